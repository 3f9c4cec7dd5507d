// Decode-sized product (M <= 64 tokens) on the tensor core with split-K.
//
// At decode sizes the layer is bound by the bytes of W it streams; 2:4 slabs
// carry 1.125 bytes per weight instead of 2, which is where PATCH's hybrid
// kernel earns its speed (abstract of "PATCH: Learnable Tile-level Hybrid
// Sparsity for LLMs"). This kernel is a streaming engine: four persistent
// CTAs per SM (independent issue loops; one loop cannot issue slabs as fast
// as HBM delivers them) walk a cost-balanced list of units (strip s, K-part
// p); warp 0 keeps the stages' slab records in flight as 2-D TMA boxes over
// the packed bytes (with an L2 evict-first hint: each is read once per call)
// plus the X box of M rounded up to 16 tokens, warp 1 runs them through
// tcgen05.mma / .mma.sp with N = that token count into a TMEM accumulator,
// and an epilogue warpgroup drains it, writing each unit's fp32 partial
// (128 rows x the tokens, token-major so a warp's accesses are coalesced) to
// a workspace. The CTA that finishes the last part of a strip (per-strip
// arrival counter) sums the strip's partials in part order, so the result
// does not depend on which CTA finishes first, writes bf16 Y and re-arms the
// counter for the next call.
//
// Two instances: up to 16 tokens (two stages and two 16-column accumulators
// per CTA) and up to 64 (two stages and one 64-column accumulator: four CTAs
// then fit the SM's 512 TMEM columns, and while one CTA's MMAs wait for its
// epilogue the other three keep streaming).
#include "kernels.cuh"

namespace patch {

namespace {

constexpr int kThreads = 64 + 128;      // producer warp, MMA warp, one epilogue warpgroup
constexpr int kStageA = 18432;          // 16 KB dense, or 8 KB values + 2 KB metadata

constexpr int tmem_cols_for(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512; }

// BN tokens per MMA, CTAS resident CTAs per SM, STAGES slab stages and ACCS
// TMEM accumulators per CTA (with one, the MMAs of the next unit wait for the
// epilogue to read the last one; the other CTAs on the SM keep streaming).
template <int BN, int CTAS, int STAGES, int ACCS>
struct DecodeCfg {
    static constexpr int kStageX = BN * 128;  // up to BN rows of 128 bytes, 128-byte swizzled
    static constexpr int kStageBytes = kStageA + kStageX;
    static constexpr int kSmemData = STAGES * kStageBytes;
    static constexpr int kSmemBytes = kSmemData + 1024 + 256;
    static constexpr int kECol = ACCS * BN;   // metadata columns after the accumulators
    static constexpr int kTmemCols = tmem_cols_for(kECol + 4);
    // tokens the split-K sum holds in registers at once
    static constexpr int kRed = CTAS > 2 && BN > 32 ? 32 : BN;
    static_assert(ACCS == 1 || ACCS == 2, "one or two accumulators");
    static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
    static_assert(kECol + 4 <= kTmemCols && kTmemCols * CTAS <= 512, "TMEM columns of the resident CTAs");
    static_assert(CTAS * (kSmemBytes + 1024) <= 228 * 1024, "shared memory of the resident CTAs");
};

// Named barrier of the epilogue warpgroup.
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int BN, int CTAS, int STAGES, int ACCS>
__global__ void __launch_bounds__(kThreads, CTAS)
    hybrid_decode_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
    using Cfg = DecodeCfg<BN, CTAS, STAGES, ACCS>;
    constexpr int kBN = BN, kStages = STAGES, kStageBytes = Cfg::kStageBytes;
    constexpr int kSmemData = Cfg::kSmemData, kECol = Cfg::kECol, kTmemCols = Cfg::kTmemCols;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* acc_full = bars + 2 * kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_full + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // token columns in use: M rounded up to the MMA's N granule of 16; the X
    // box (encoded by the host) and every MMA cover just these
    const int n_tok = min(kBN, (a.M + 15) & ~15);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);  // the four warps of the warpgroup draining it
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto raise = [&]() {
        *abort_flag = 1;
        atomicCAS(a.status, 0, kStatusTimeout);
    };
    const int w_begin = a.work_off[blockIdx.x];
    const int w_end = a.work_off[blockIdx.x + 1];
    // part p of a strip covers chunks [p*KC/P, (p+1)*KC/P), i.e. slabs from 2x that
    auto part_range = [](const LinDesc& L, int p, int& b0, int& b1) {
        const int P = BN == kDecodeBN ? L.P : L.PW;
        b0 = 2 * (int)(((int64_t)p * L.KC) / P);
        b1 = min(L.KB, 2 * (int)(((int64_t)(p + 1) * L.KC) / P));
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int it = w_begin; it < w_end && ok; ++it) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int P = BN == kDecodeBN ? L.P : L.PW;
                const int s = lu / P, p = lu % P;
                int b0, b1;
                part_range(L, p, b0, b1);
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const uint32_t* mrow = L.meta + (size_t)s * L.KC;
                const uint64_t pol_w = policy_evict_first();  // weights are read once per call
                const CUtensorMap* tmap_x = &maps.x[l];
                uint32_t d_next = b0 < b1 ? trow[b0] : 0u;
                for (int b = b0; b < b1; ++b) {
                    const uint32_t d = d_next;
                    if (b + 1 < b1) d_next = trow[b + 1];  // fetched one slab ahead
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const bool sp = d & kSlabSparse, first = d & kSlabFirst;
                    const uint32_t bytes_a = sp ? kSparseValBytes : kDenseSlabBytes;
                    uint8_t* st = smem + stage * kStageBytes;
                    mbar_arrive_expect_tx(&full[stage], bytes_a + (first ? kMetaBytes : 0) + (uint32_t)n_tok * 128u);
                    // the packed bytes viewed as 128-byte rows: one 2-D box per record
                    tma_load_2d_hint(st, sp ? &maps.a8[l] : &maps.a16[l], &full[stage], 0,
                                     (int)(slab_offset_bytes(d) >> 7), pol_w);
                    if (first)
                        tma_load_2d_hint(st + kSparseValBytes, &maps.e[l], &full[stage], 0, (int)(mrow[b >> 1] >> 3),
                                         pol_w);
                    tma_load_2d(st + kStageA, tmap_x, &full[stage], b * kSlabK, 0);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            int st = stage;
            uint32_t ph = phase;
            for (int i = 0; i < kStages && i < issued; ++i) {
                if (--st < 0) {
                    st = kStages - 1;
                    ph ^= 1u;
                }
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&full[st], ph) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc_d = idesc_bf16(128, n_tok, false);
            const uint32_t idesc_s = idesc_bf16(128, n_tok, true);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any_mma = false;
            bool ready = false;  // full[stage] already seen complete by the look-ahead
            int t = 0;
            for (int it = w_begin; it < w_end && ok; ++it, ++t) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int P = BN == kDecodeBN ? L.P : L.PW;
                const int s = lu / P, p = lu % P;
                int b0, b1;
                part_range(L, p, b0, b1);
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const int acc = t % ACCS;
                if (!mbar_wait(&acc_empty[acc], ((t / ACCS) & 1) ^ 1u, abort_flag)) {
                    raise();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
                uint32_t d = b0 < b1 ? trow[b0] : 0u;
                for (int b = b0; b < b1; ++b) {
                    // the record comes one slab ahead and the next stage is
                    // tested before this slab's MMAs (see the pair kernel)
                    if (!ready && !mbar_wait(&full[stage], phase, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const uint32_t d_next = b + 1 < b1 ? trow[b + 1] : 0u;
                    int next = stage + 1;
                    uint32_t next_phase = phase;
                    if (next == kStages) {
                        next = 0;
                        next_phase ^= 1u;
                    }
                    ready = mbar_test_wait(&full[next], next_phase);
                    const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
                    const uint32_t x_addr = a_addr + kStageA;
                    const uint32_t first_mma = (b == b0) ? 0u : 1u;
                    if (d & kSlabSparse) {
                        if (d & kSlabFirst)
                            tc_cp_128x128b(tmem_base + kECol,
                                           smem_desc(a_addr + kSparseValBytes, 16, 128, kLayoutNone));
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 512, kLayoutSw64);
                            const uint64_t bd = smem_desc(x_addr + i * 64, 16, 1024, kLayoutSw128);
                            const uint32_t ecol = kECol + (b & 1) * 2 + i;
                            mma_sp_bf16(d_tmem, ad, bd, idesc_s | (ecol & 1u), tmem_base + (ecol & ~1u),
                                        first_mma | (uint32_t)i);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 1024, kLayoutSw128);
                            const uint64_t bd = smem_desc(x_addr + i * 32, 16, 1024, kLayoutSw128);
                            mma_bf16(d_tmem, ad, bd, idesc_d, first_mma | (uint32_t)i);
                        }
                    }
                    any_mma = true;
                    tc_commit(&empty[stage]);
                    stage = next;
                    phase = next_phase;
                    d = d_next;
                }
                if (!ok) break;
                tc_commit(&acc_full[acc]);
            }
            if (*abort_flag && any_mma) {
                tc_commit(drain);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---------------- epilogue: warps 2..5, one TMEM lane quadrant each ----------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;
        constexpr int kLeader = 64;  // first thread of the warpgroup
        int t = 0;
        for (int it = w_begin; it < w_end; ++it, ++t) {
            const int acc = t % ACCS;
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const LinDesc& L = a.lins[l];
            const int P = BN == kDecodeBN ? L.P : L.PW;
            const int s = lu / P, p = lu % P;
            if (!mbar_wait(&acc_full[acc], (t / ACCS) & 1, abort_flag)) {
                if (lane == 0) raise();
                break;
            }
            tc_fence_after();
            __nv_bfloat16* yc = a.Y[l] + (size_t)s * kStrip + row;
            // this unit's partial, workspace[s][p][token][row], for the M
            // tokens only: a warp's stores and loads of one token cover 128
            // contiguous bytes
            float* dst = P > 1 ? a.partial[l] + ((size_t)s * P + p) * kBN * 128 + row : nullptr;
            const int cols = n_tok;
            // 16 columns at a time: Y directly when the strip is one unit,
            // else the partial
#pragma unroll
            for (int c0 = 0; c0 < kBN; c0 += 16) {
                if (c0 >= cols) break;
                uint32_t v[16];
                tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN + c0), v);
                tc_wait_ld();
                if (P == 1) {
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c0 + c < a.M) yc[(size_t)(c0 + c) * L.N] = __float2bfloat16_rn(__uint_as_float(v[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c0 + c < a.M) __stcg(dst + (c0 + c) * 128, __uint_as_float(v[c]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            if (P == 1) continue;
            epi_bar();
            if ((int)threadIdx.x == kLeader) {
                // the barrier orders the warpgroup's stores before this fence,
                // which releases them with the arrival
                __threadfence();
                const unsigned old = atomicAdd(&a.counters[l][s], 1u);
                *last_flag = (old == (unsigned)(P - 1));
            }
            epi_bar();
            if (*last_flag) {
                __threadfence();
                // sum the parts in part order; all of one part's loads of a
                // chunk of kRed tokens are in flight together
                constexpr int kRed = Cfg::kRed;
#pragma unroll
                for (int c0 = 0; c0 < kBN; c0 += kRed) {
                    if (c0 >= cols) break;
                    float sum[kRed];
#pragma unroll
                    for (int c = 0; c < kRed; ++c) sum[c] = 0.f;
                    const float* src = a.partial[l] + (size_t)s * P * kBN * 128 + c0 * 128 + row;
                    for (int pp = 0; pp < P; ++pp, src += kBN * 128) {
                        float v[kRed];
#pragma unroll
                        for (int c = 0; c < kRed; ++c) v[c] = c0 + c < a.M ? __ldcg(src + c * 128) : 0.f;
#pragma unroll
                        for (int c = 0; c < kRed; ++c) sum[c] += v[c];
                    }
#pragma unroll
                    for (int c = 0; c < kRed; ++c)
                        if (c0 + c < a.M) yc[(size_t)(c0 + c) * L.N] = __float2bfloat16_rn(sum[c]);
                }
                if ((int)threadIdx.x == kLeader) a.counters[l][s] = 0u;  // re-armed for the next call
            }
            // the flag is rewritten only after the next unit's first barrier,
            // which every thread reaches after reading it here
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace

// BN = 16: M <= 16, four CTAs per SM, two stages and two accumulators each.
// BN = kDecodeWideBN: 16 < M <= kDecodeWideBN, kDecodeWideCtasPerSm CTAs per SM
// (the stage and accumulator counts are macros so that other splits of the
// SM's shared memory and TMEM can be measured).
#ifndef PATCH_DECODE_WIDE_STAGES
#define PATCH_DECODE_WIDE_STAGES 2
#endif
#ifndef PATCH_DECODE_WIDE_ACCS
#define PATCH_DECODE_WIDE_ACCS 1
#endif
using Narrow = DecodeCfg<kDecodeBN, kDecodeCtasPerSm, 2, 2>;
using Wide = DecodeCfg<kDecodeWideBN, kDecodeWideCtasPerSm, PATCH_DECODE_WIDE_STAGES, PATCH_DECODE_WIDE_ACCS>;
#define PATCH_DECODE16 hybrid_decode_kernel<kDecodeBN, kDecodeCtasPerSm, 2, 2>
#define PATCH_DECODE_WIDE \
    hybrid_decode_kernel<kDecodeWideBN, kDecodeWideCtasPerSm, PATCH_DECODE_WIDE_STAGES, PATCH_DECODE_WIDE_ACCS>

cudaError_t decode_prepare() {
    cudaError_t e = cudaFuncSetAttribute(PATCH_DECODE16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Narrow::kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(PATCH_DECODE_WIDE, cudaFuncAttributeMaxDynamicSharedMemorySize, Wide::kSmemBytes);
}

cudaError_t launch_decode(const GroupMaps& maps, const GroupArgs& a, int grid, int bn, cudaStream_t st) {
    if (bn == kDecodeWideBN)
        PATCH_DECODE_WIDE<<<grid, kThreads, Wide::kSmemBytes, st>>>(maps, a);
    else
        PATCH_DECODE16<<<grid, kThreads, Narrow::kSmemBytes, st>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace patch
