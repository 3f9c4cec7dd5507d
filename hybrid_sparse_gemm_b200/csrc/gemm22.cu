// Hybrid dense / 2:4 GEMM on CTA pairs with two strips per CTA:
// Y = X . (W (.) Mask)^T.
//
// Same method as the other tensor-core kernels (dense slabs on tcgen05.mma,
// 2:4 slabs on tcgen05.mma.sp; PATCH abstract, "PATCH: Learnable Tile-level
// Hybrid Sparsity for LLMs"), arranged so that each activation tile feeds twice
// the tensor work. A cluster of two CTAs owns a strip quad (strips 4c .. 4c+3)
// and a block of 240 tokens. Every 64-column slab issues two 256-row MMAs
// (cta_group::2), one per strip pair: strips (4c, 4c+1) into accumulator 0 and
// (4c+2, 4c+3) into accumulator 1. CTA r holds strips 4c+r and 4c+2+r
// (operand A) and tokens [r*N/2, (r+1)*N/2) of the block (operand B), so each
// activation byte loaded from L2 serves 512 weight rows. Each strip pair has
// its own issuing thread, so the tensor pipe is fed by two instruction
// streams (one thread alone cannot issue 2:4 slabs as fast as they execute).
//
// TMEM (512 columns per CTA): accumulator 0 in columns [0, 240), accumulator
// 1 in [256, 496), the 2:4 metadata of each strip in four columns at 240 and
// 248. The accumulators are single-buffered: a tile's MMAs start once the
// previous tile has been drained, while the producers keep filling the ring.
//
// Partner strips (the strips at pair positions 2p and 2p+1 of the member's
// pair order) load the same kind of record at every slab (the packed
// format's dense images stand in for 2:4 slabs whose partner is dense), so
// one MMA instruction always covers both halves of a pair. Positions past the
// end of the weight are replaced by duplicates whose results are not stored.
#include "kernels.cuh"
#include "pair.cuh"

namespace patch {

namespace {

#ifndef PATCH_GEMM22_PRODUCERS
#define PATCH_GEMM22_PRODUCERS 4
#endif
constexpr int kProducers = PATCH_GEMM22_PRODUCERS;  // TMA-issuing warps (stages dealt round robin)
constexpr int kMmaWarp = kProducers;            // MMA issuers (leader CTA), one per strip pair;
constexpr int kMmaWarps = 2;                    // the first also owns TMEM
constexpr int kEpiWarp0 = kMmaWarp + kMmaWarps;
constexpr int kEpiWarps = 16;                   // per accumulator, two warps per TMEM lane quarter
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kBN = kGemm22BN;                  // tokens per tile (both CTAs)
constexpr int kHalfN = kBN / 2;                 // token rows of operand B per CTA
constexpr int kStageX = kHalfN * 128;           // 15 KB of activations per slab
#ifndef PATCH_GEMM22_RING
#define PATCH_GEMM22_RING 218112
#endif
constexpr int kRing = PATCH_GEMM22_RING;        // shared-memory ring the stages are placed in, in order
constexpr int kQ = 8;                           // per-stage barriers: more than the stages that fit in the ring
// Largest two-slab stage; larger ones are cut into one-slab stages. The pure
// 2:4 instance keeps two-slab stages (66 KB); the general instance cuts every
// chunk, which keeps six or more stages in flight to cover the load latency.
constexpr uint32_t kMaxStagePure = 70 * 1024;
#ifndef PATCH_GEMM22_MAX_STAGE
#define PATCH_GEMM22_MAX_STAGE 40 * 1024
#endif
constexpr uint32_t kMaxStageMixed = PATCH_GEMM22_MAX_STAGE;
// smallest stage: one 2:4 slab of each strip and its activation tile
constexpr int kMinStage = 2 * kSparseValBytes + kStageX;
static_assert(kRing % 1024 == 0 && kStageX % 1024 == 0 && kMetaBytes % 1024 == 0,
              "every record starts 1024-byte aligned (128-byte swizzle atoms)");
static_assert(kRing / kMinStage + 2 <= kQ, "stages in flight stay within the barrier window");
// Each producer warp copies the slab records and metadata block offsets of
// its current tile's two strips into shared memory, so that no stage waits
// on a table read from L2. Weights with more than kTabKB slabs per strip read
// the tables from global memory instead.
constexpr int kTabKB = 256;                     // K up to 16384
constexpr int kTabWords = 2 * kTabKB + 2 * (kTabKB / 2);
constexpr int kSmemData = kRing;
constexpr int kSmemTab = kProducers * kTabWords * 4;
constexpr int kSmemBytes = kSmemData + kSmemTab + 1024 + 512;
static_assert(kSmemBytes <= 232448, "fits the 227 KB of shared memory a CTA may use");
constexpr int kAcc1 = 256;                      // first column of accumulator 1
constexpr int kECol0 = kBN;                     // metadata columns of strip pair 0
constexpr int kECol1 = kBN + 8;                 // ... and of strip pair 1
constexpr int kTmemCols = 512;
static_assert(kECol1 + 4 <= kAcc1, "metadata columns fit between the accumulators");

// Token tiles: the MB = ceil(M / kBN) tiles share M's ceil(M / 16)
// 16-token granules as evenly as possible (so no tile is a sliver that
// streams a strip quad's weights for a few tokens): a.tile_gran each and one
// more for the first a.tile_extra tiles (computed on the host). Tile j starts
// at token tile_start(j) and its MMAs have N = tile_tokens(j), a multiple of
// 16 and at most kBN; the last tile's N may reach past M (those columns are
// never stored).
__device__ __forceinline__ int tile_start(const GroupArgs& a, int j) {
    return 16 * (j * a.tile_gran + min(j, a.tile_extra));
}
__device__ __forceinline__ int tile_tokens(const GroupArgs& a, int j) {
    return 16 * (a.tile_gran + (j < a.tile_extra ? 1 : 0));
}

__device__ __forceinline__ uint32_t rec_bytes(uint32_t d) {
    return (d & kSlabSparse) ? kSparseValBytes : kDenseSlabBytes;
}

// A chunk is two 64-column slabs (one for an odd last chunk) of a strip. A
// stage holds both strips' records of one chunk, or of one slab of it when
// the two-slab stage would exceed the instance's limit (kMaxStagePure or
// kMaxStageMixed: more, smaller stages in the ring cover more of the load
// latency), plus the activation tiles of those slabs. A strip's part of a
// stage: its slab records back to back, then, in the stage that holds the
// chunk's first slab, the chunk's 2 KB metadata block when either slab runs
// on the sparse MMA (the metadata columns it fills in TMEM serve both slabs).
struct Chunk {
    uint32_t d0, d1;  // gemm-table records of the chunk's slabs
    int n;            // slabs in the chunk (1 or 2)
    __device__ __forceinline__ uint32_t rec(int i) const { return i ? d1 : d0; }
    __device__ __forceinline__ bool sparse() const {
        return ((d0 | (n > 1 ? d1 : 0u)) & kSlabSparse) != 0;
    }
    // record bytes of slabs [f, f + m)
    __device__ __forceinline__ uint32_t recs(int f, int m) const {
        return m > 1 ? rec_bytes(d0) + rec_bytes(d1) : rec_bytes(rec(f));
    }
    __device__ __forceinline__ bool meta_in(int f) const { return f == 0 && sparse(); }
    // this strip's bytes in the stage of slabs [f, f + m)
    __device__ __forceinline__ uint32_t bytes(int f, int m) const {
        return recs(f, m) + (meta_in(f) ? (uint32_t)kMetaBytes : 0u);
    }
    // kinds of this strip's slabs in the stage: bit 0 first slab 2:4, bit 1
    // second slab 2:4, bit 2 the chunk's metadata block is in the stage
    __device__ __forceinline__ uint32_t kinds(int f, int m) const {
        return (rec(f) & kSlabSparse) | (m > 1 ? (d1 & kSlabSparse) << 1 : 0u) | (meta_in(f) ? 4u : 0u);
    }
};

__device__ __forceinline__ Chunk load_chunk(const uint32_t* t, int c, int KB) {
    Chunk k;
    k.n = (2 * c + 1 < KB) ? 2 : 1;
    k.d0 = t[2 * c];
    k.d1 = k.n > 1 ? t[2 * c + 1] : 0u;
    return k;
}

// A weight whose every slab runs on the sparse MMA (a pure 2:4 weight, the
// MaskLLM end of the hybrid range) has a packed layout with no dense records
// and no dense images: strip s's compressed slab b sits at (s*KB + b) * 8 KB,
// and the metadata block of its chunk c right after all values, at
// S*KB*8 KB + (s*KC + c) * 2 KB. The kernel instance for such weights
// computes the records instead of reading the tables.
__device__ __forceinline__ Chunk pure_chunk(int s, int c, int KB) {
    Chunk k;
    k.n = (2 * c + 1 < KB) ? 2 : 1;
    const uint32_t v = (uint32_t)(((size_t)s * KB + 2 * c) * (kSparseValBytes / 16));
    k.d0 = (v << 2) | kSlabSparse;
    k.d1 = k.n > 1 ? ((v + kSparseValBytes / 16) << 2) | kSlabSparse : 0u;
    return k;
}
__device__ __forceinline__ uint32_t pure_meta(int S, int KB, int KC, int s, int c) {
    return (uint32_t)(((size_t)S * KB * kSparseValBytes + ((size_t)s * KC + c) * kMetaBytes) / 16);
}

// What the MMA issuers need of a stage, written by the leader CTA's producer
// that loads it, before the stage's loads are counted on its full barrier
// (so the issuers' wait on that barrier also orders this read):
//   x ring offset, y bytes of strip pair 0's part | strip pair 1's << 16,
//   z kinds of strip pair 0 | strip pair 1's << 8, w slabs (1 or 2) | first
//   slab's half of the chunk << 2 | first stage of the tile << 3 | last << 4.
struct StageDesc {
    uint32_t off, bytes, kinds, flags;
};

// Stages are placed one after another in a ring of kRing bytes; a stage that
// does not fit before the end starts again at 0. `pos` counts bytes placed so
// far (including skipped ends); returns the ring offset of this stage.
struct Ring {
    uint32_t pos = 0, off = 0;
    __device__ __forceinline__ uint32_t place(uint32_t size) {
        if (off + size > (uint32_t)kRing) {
            pos += (uint32_t)kRing - off;
            off = 0;
        }
        const uint32_t at = off;
        pos += size;
        off += size;
        return at;
    }
};

// One strip pair's MMAs for one slab: 4 dense K=16 MMAs, or 2 sparse K=32
// MMAs reading the metadata columns of this slab's half of the chunk.
__device__ __forceinline__ void issue_slab(uint32_t d, int half, bool first, uint32_t a_addr, uint32_t b_addr,
                                           uint32_t d_tmem, uint32_t e_col, uint32_t idesc_d, uint32_t idesc_s) {
    if (d & kSlabSparse) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 512, kLayoutSw64);
            const uint64_t bd = smem_desc(b_addr + i * 64, 16, 1024, kLayoutSw128);
            const uint32_t ecol = e_col + (uint32_t)(half * 2 + i);
            mma2_sp_bf16(d_tmem, ad, bd, idesc_s | (ecol & 1u), ecol & ~1u, !(first && i == 0));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 1024, kLayoutSw128);
            const uint64_t bd = smem_desc(b_addr + i * 32, 16, 1024, kLayoutSw128);
            mma2_bf16(d_tmem, ad, bd, idesc_d, !(first && i == 0));
        }
    }
}

template <bool kPure24>
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_gemm22_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint32_t* tabs = reinterpret_cast<uint32_t*>(smem + kSmemData);  // [warp][kTabWords]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData + kSmemTab);
    uint64_t* full = bars;                       // [kQ] leader: both CTAs' bytes of stage g (at g % kQ)
    uint64_t* empty = full + kQ;                 // [kQ] every CTA: stage g consumed by both issuers
    uint64_t* acc_full = empty + kQ;             // [2] both CTAs: accumulator h ready
    uint64_t* acc_empty = acc_full + 2;          // [2] leader: the 16 epilogue warps of accumulator h drained it
    uint64_t* drain = acc_empty + 2;             // [2]
    StageDesc* sdesc = reinterpret_cast<StageDesc*>(drain + 2);  // [kQ] leader: stage g at g % kQ
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sdesc + kQ);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t pr = cluster_rank();          // CTA within the pair (0 = leader)
    const int cl = blockIdx.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQ; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kMmaWarps);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&acc_full[h], 1);
            mbar_init(&acc_empty[h], kEpiWarps);  // its 8 epilogue warps in each of the 2 CTAs
            mbar_init(&drain[h], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc2(tmem_slot, kTmemCols);
        tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers of both CTAs initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto raise = [&]() {
        *abort_flag = 1;
        atomicCAS(a.status, 0, kStatusTimeout);
    };
    // Pair position of the strip this CTA loads for strip pair h of quad c
    // of member L (the tables L.gemm and L.pmeta have their rows in this
    // order; with pure 2:4 weights it is the strip order). Missing positions
    // fall back to one whose partner relation is kept, so both halves of
    // every MMA stay one kind.
    auto pos_of = [&](const LinDesc& L, int c, int h) {
        const int S = L.S;
        int pos = 4 * c + 2 * h + (int)pr;
        if (pos >= S) pos = 4 * c + 2 * h;
        if (pos >= S) pos = 4 * c + (int)pr;
        if (pos >= S) pos = 4 * c;
        return pos;
    };

    const int w_begin = a.work_off[cl];
    const int w_end = a.work_off[cl + 1];
    // Warp-cooperative copy of n table entries into shared memory; returns the
    // shared copy, or the global table itself when it does not fit.
    auto stage_table = [&](uint32_t* dst, const uint32_t* src, int n) -> const uint32_t* {
        if (n > kTabKB) return src;
        for (int i = lane; i < n; i += 32) dst[i] = src[i];
        return dst;
    };

    if (warp < kProducers) {
        {
            // ---------------- producers (both CTAs) ----------------
            // Every producer walks the whole stage sequence to place each stage
            // in the ring; it loads the stages g with g % kProducers == me.
            // Before loading, the stages that last used those ring bytes must
            // have been consumed (in order, so waiting for the latest suffices).
            const int me = warp;
            Ring ring;
            uint32_t hist[kQ];   // ring positions where the last kQ stages started
            int g = 0;
            int my_last = -1;    // sequence index of the last stage this producer loaded
            bool ok = true;
            // every strip quad of a member reads the same activation tiles, so
            // they are kept in L2 over the weight records (each read by one
            // wave of token tiles)
            const uint64_t pol_x = policy_evict_last();
            for (int it = w_begin; it < w_end && ok; ++it) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int c = lu / a.MB, j = lu % a.MB;
                const int KB = L.KB, KC = L.KC;
                const int s0 = pos_of(L, c, 0), s1 = pos_of(L, c, 1);
                uint32_t* tab = tabs + warp * kTabWords;
                const uint32_t *t0 = nullptr, *t1 = nullptr, *m0 = nullptr, *m1 = nullptr;
                if (!kPure24) {
                    t0 = stage_table(tab, L.gemm + (size_t)s0 * KB, KB);
                    t1 = stage_table(tab + kTabKB, L.gemm + (size_t)s1 * KB, KB);
                    m0 = stage_table(tab + 2 * kTabKB, L.pmeta + (size_t)s0 * KC, KB > kTabKB ? kTabKB + 1 : KC);
                    m1 = stage_table(tab + 2 * kTabKB + kTabKB / 2, L.pmeta + (size_t)s1 * KC,
                                     KB > kTabKB ? kTabKB + 1 : KC);
                    __syncwarp();
                }
                const CUtensorMap* tm_x = &maps.x[l];
                const int tok = tile_start(a, j) + (int)pr * (tile_tokens(a, j) >> 1);
                for (int kc = 0, part = 0; lane == 0 && kc < KC; ++g) {
                    const Chunk k0 = kPure24 ? pure_chunk(s0, kc, KB) : load_chunk(t0, kc, KB);
                    const Chunk k1 = kPure24 ? pure_chunk(s1, kc, KB) : load_chunk(t1, kc, KB);
                    const bool split = k0.n == 2 && k0.bytes(0, 2) + k1.bytes(0, 2) + 2 * kStageX > (kPure24 ? kMaxStagePure : kMaxStageMixed);
                    const int f = split ? part : 0, m = split ? 1 : k0.n;
                    const int kc_now = kc;
                    if (!split || part == 1) {
                        ++kc;
                        part = 0;
                    } else {
                        part = 1;
                    }
                    const uint32_t size = k0.bytes(f, m) + k1.bytes(f, m) + (uint32_t)m * kStageX;
                    const uint32_t off = ring.place(size);
                    hist[g % kQ] = ring.pos - size;
                    if (g % kProducers != me) continue;
                    if (ring.pos > (uint32_t)kRing) {
                        const uint32_t need = ring.pos - (uint32_t)kRing;
                        int jl = -1;
                        for (int jj = g - 1; jj >= 0 && jj > g - kQ; --jj)
                            if (hist[jj % kQ] < need) {
                                jl = jj;
                                break;
                            }
                        if (jl >= 0 && !mbar_wait(&empty[jl % kQ], (uint32_t)((jl / kQ) & 1), abort_flag)) {
                            raise();
                            ok = false;
                            break;
                        }
                    }
                    const uint32_t bar = map_to_rank(smem_u32(&full[g % kQ]), 0);
                    if (pr == 0) {
                        StageDesc sd;
                        sd.off = off;
                        sd.bytes = k0.bytes(f, m) | (k1.bytes(f, m) << 16);
                        sd.kinds = k0.kinds(f, m) | (k1.kinds(f, m) << 8);
                        sd.flags = (uint32_t)m | ((uint32_t)f << 2) | ((kc_now == 0 && f == 0) ? 8u : 0u) |
                                   (kc >= KC ? 16u : 0u);
                        sdesc[g % kQ] = sd;
                        mbar_arrive_expect_tx(&full[g % kQ], 2u * size);
                    }
                    uint32_t dst = smem_u32(smem) + off;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const Chunk k = h ? k1 : k0;
                        const uint32_t da = k.rec(f), db = k.d1;
                        // both slabs in one copy when their records are adjacent
                        // and of one kind (a 2:4 pair is one 128-row box, a dense
                        // pair one 256-row box)
                        const bool joint = m == 2 && ((da ^ db) & kSlabSparse) == 0 &&
                                           slab_offset_bytes(db) == slab_offset_bytes(da) + rec_bytes(da);
                        if (joint) {
                            tma_load_2d_pair(dst, (da & kSlabSparse) ? &maps.a16[l] : &maps.a32[l], bar, 0,
                                             (int)(slab_offset_bytes(da) >> 7));
                        } else {
                            tma_load_2d_pair(dst, (da & kSlabSparse) ? &maps.a8[l] : &maps.a16[l], bar, 0,
                                             (int)(slab_offset_bytes(da) >> 7));
                            if (m > 1)
                                tma_load_2d_pair(dst + rec_bytes(da), (db & kSlabSparse) ? &maps.a8[l] : &maps.a16[l],
                                                 bar, 0, (int)(slab_offset_bytes(db) >> 7));
                        }
                        if (k.meta_in(f)) {
                            const uint32_t mrow =
                                kPure24 ? pure_meta(L.S, KB, KC, h ? s1 : s0, kc_now) : (h ? m1 : m0)[kc_now];
                            tma_load_2d_pair(dst + k.recs(f, m), &maps.e[l], bar, 0, (int)(mrow >> 3));
                        }
                        dst += k.bytes(f, m);
                    }
                    for (int i = 0; i < m; ++i)
                        tma_load_2d_pair_hint(dst + i * kStageX, tm_x, bar, (2 * kc_now + f + i) * kSlabK, tok, pol_x);
                    my_last = g;
                }
                // the whole warp moves on to the next tile (or stops) with lane 0
                ok = __shfl_sync(0xffffffffu, ok, 0);
                __syncwarp();
            }
            if (pr == 0 && lane == 0) {
                // Bounded wait for the loads of my stages among the last kQ of
                // the sequence, whatever the abort flag says, so none lands
                // after the cluster exits. (Earlier stages were consumed before
                // the ring bytes were reused, and no stage gg + kQ exists to
                // have moved the barrier past the phase waited for.)
                for (int gg = g - kQ; gg <= my_last; ++gg) {
                    if (gg < 0 || gg % kProducers != me) continue;
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&full[gg % kQ], (uint32_t)((gg / kQ) & 1)) &&
                           globaltimer() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp < kMmaWarp + kMmaWarps) {
        if (lane == 0 && pr == 0) {
            // ---------------- MMA issuers (leader CTA), one per strip pair ----------------
            // Both read every stage; a stage's ring bytes are free once both
            // have committed it. Two issuing threads keep the tensor pipe fed
            // while either one waits on a barrier or computes descriptors. The
            // stage layout comes from the descriptor its producer wrote.
            const int h = warp - kMmaWarp;
            const uint32_t d_tmem = tmem_base + (uint32_t)(h * kAcc1);
            const uint32_t e_col = tmem_base + (uint32_t)(h ? kECol1 : kECol0);
            const uint32_t ring0 = smem_u32(smem);
            int g = 0;
            bool ok = true, any_mma = false;
            int t = 0;
            for (int it = w_begin; it < w_end && ok; ++it, ++t) {
                const int j = (a.work[it] & kUnitMask) % a.MB;
                const int nt = tile_tokens(a, j);
                const uint32_t idesc_d = idesc_bf16(256, nt, false);
                const uint32_t idesc_s = idesc_bf16(256, nt, true);
                if (!mbar_wait(&acc_empty[h], (t & 1) ^ 1u, abort_flag)) {
                    raise();
                    break;
                }
                tc_fence_after();
                for (bool last = false; !last; ++g) {
                    if (!mbar_wait(&full[g % kQ], (uint32_t)((g / kQ) & 1), abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const StageDesc sd = sdesc[g % kQ];
                    const uint32_t b0 = sd.bytes & 0xFFFFu, b1 = sd.bytes >> 16;
                    const uint32_t kd = h ? (sd.kinds >> 8) & 0xFFu : sd.kinds & 0xFFu;
                    const int m = (int)(sd.flags & 3u), f = (int)((sd.flags >> 2) & 1u);
                    const bool first = (sd.flags & 8u) != 0;
                    last = (sd.flags & 16u) != 0;
                    const uint32_t a_addr = ring0 + sd.off + (h ? b0 : 0u);
                    const uint32_t b_addr = ring0 + sd.off + b0 + b1;
                    const uint32_t r0 = (kd & 1u) ? (uint32_t)kSparseValBytes : (uint32_t)kDenseSlabBytes;
                    const uint32_t r1 = m > 1 ? ((kd & 2u) ? (uint32_t)kSparseValBytes : (uint32_t)kDenseSlabBytes) : 0u;
                    if (kd & 4u) cp2_128x128b(e_col, smem_desc(a_addr + r0 + r1, 16, 128, kLayoutNone));
                    issue_slab(kd & 1u, f, first, a_addr, b_addr, d_tmem, e_col, idesc_d, idesc_s);
                    if (m > 1)
                        issue_slab((kd >> 1) & 1u, 1, false, a_addr + r0, b_addr + kStageX, d_tmem, e_col, idesc_d,
                                   idesc_s);
                    any_mma = true;
                    commit2_mask(&empty[g % kQ], 3);
                }
                if (!ok) break;
                commit2_mask(&acc_full[h], 3);
            }
            if (*abort_flag && any_mma) {
                commit2_local(&drain[h]);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&drain[h], 0) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---------------- epilogue (16 warps, both CTAs) ----------------
        const int h = (warp - kEpiWarp0) >> 3;   // accumulator (strip pair) this warp drains
        const int ch = ((warp - kEpiWarp0) >> 2) & 1;  // this warp takes every other 32-token chunk
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        int t = 0;
        for (int it = w_begin; it < w_end; ++it, ++t) {
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const int N = a.lins[l].N;
            const int c = lu / a.MB, j = lu % a.MB;
            const int pos = 4 * c + 2 * h + (int)pr;  // pair position of this CTA's strip
            const bool store = pos < a.lins[l].S;
            const int s = store ? a.lins[l].order[pos] : 0;
            const int nt = tile_tokens(a, j);
            const int tok0 = tile_start(a, j);
            const int mrem = a.M - tok0;  // tokens of the tile that exist
            if (!mbar_wait(&acc_full[h], t & 1, abort_flag)) {
                if (lane == 0) raise();
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kAcc1);
            __nv_bfloat16* yc = a.Y[l] + (size_t)tok0 * N + (size_t)s * kStrip + q * 32 + lane;
            if (store) {
                // 32-column chunks, alternating between the two warps of a lane
                // quarter (the last chunk of a 240-token tile has 16 columns).
#pragma unroll 1
                for (int c0 = 32 * ch; c0 < nt; c0 += 64) {
                    uint32_t v[32];
                    const int cols = nt - c0 >= 32 ? 32 : 16;
                    if (cols == 32)
                        tmem_ld_32x32b_x32(taddr + c0, v);
                    else
                        tmem_ld_32x32b_x16(taddr + c0, v);
                    tc_wait_ld();
                    if (c0 + cols <= mrem) {
                        // Lanes 2i and 2i+1 hold rows 2i and 2i+1 of Y's columns;
                        // one swap per two tokens lets each lane store both rows'
                        // values of one token as a 4-byte pair (half the stores).
                        __nv_bfloat16* yq = yc - lane + (lane & ~1);
                        const bool odd = lane & 1;
#pragma unroll
                        for (int cc = 0; cc < 32; cc += 2) {
                            if (cc >= cols) break;
                            const float x0 = __uint_as_float(v[cc]), x1 = __uint_as_float(v[cc + 1]);
                            const float recv = __shfl_xor_sync(0xffffffffu, odd ? x0 : x1, 1);
                            const __nv_bfloat162 two =
                                odd ? __floats2bfloat162_rn(recv, x1) : __floats2bfloat162_rn(x0, recv);
                            *reinterpret_cast<__nv_bfloat162*>(yq + (size_t)(c0 + cc + (odd ? 1 : 0)) * N) = two;
                        }
                    } else {
#pragma unroll
                        for (int cc = 0; cc < 32; ++cc)
                            if (cc < cols && c0 + cc < mrem)
                                yc[(size_t)(c0 + cc) * N] = __float2bfloat16_rn(__uint_as_float(v[cc]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) remote_arrive(map_to_rank(smem_u32(&acc_empty[h]), 0));
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while the other may still signal it
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc2(tmem_base, kTmemCols);
    }
}

cudaLaunchConfig_t config(int clusters, cudaLaunchAttribute* attr, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = 2;
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

}  // namespace

cudaError_t gemm_prepare_wide(int* max_clusters) {
    cudaError_t e =
        cudaFuncSetAttribute(hybrid_gemm22_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(hybrid_gemm22_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = config(1, &attr, nullptr);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, hybrid_gemm22_kernel<false>, &cfg);
    if (e != cudaSuccess) return e;
    *max_clusters = n;
    return cudaSuccess;
}

cudaError_t launch_gemm22(const GroupMaps& maps, const GroupArgs& a, int clusters, bool pure24, cudaStream_t st) {
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = config(clusters, &attr, st);
    return pure24 ? cudaLaunchKernelEx(&cfg, hybrid_gemm22_kernel<true>, maps, a)
                  : cudaLaunchKernelEx(&cfg, hybrid_gemm22_kernel<false>, maps, a);
}

}  // namespace patch
