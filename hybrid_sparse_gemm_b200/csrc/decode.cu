// Decode-sized product (M <= 16 tokens) on the tensor core with split-K.
//
// At decode sizes the layer is bound by the bytes of W it streams; 2:4 slabs
// carry 1.125 bytes per weight instead of 2, which is where PATCH's hybrid
// kernel earns its speed (abstract of "PATCH: Learnable Tile-level Hybrid
// Sparsity for LLMs"). This kernel is a streaming engine: four persistent
// CTAs per SM (four independent issue loops; one loop cannot issue slabs as
// fast as HBM delivers them) walk a cost-balanced list of units (strip s,
// K-part p); warp 0 keeps kStages slab records in flight as 2-D TMA boxes
// over the packed bytes (plus the 16-token X box), warp 1 runs them through
// tcgen05.mma / .mma.sp with N = 16 into one of two TMEM accumulators, and an
// epilogue warpgroup drains them alternately, writing each unit's fp32
// partial (128 rows x 16 tokens) to a workspace. The CTA that finishes the
// last part of a strip (per-strip arrival counter) sums the strip's partials
// in part order, so the result does not depend on which CTA finishes first,
// writes bf16 Y and re-arms the counter for the next call.
#include "kernels.cuh"

namespace patch {

namespace {

constexpr int kEpiGroups = 1;           // epilogue warpgroups (units dealt round robin)
constexpr int kThreads = 64 + 128 * kEpiGroups;  // producer warp, MMA warp, epilogue
constexpr int kBN = kDecodeBN;           // tokens per MMA (M <= 16)
constexpr int kStageA = 18432;           // 16 KB dense, or 8 KB values + 2 KB metadata
constexpr int kStageX = kBN * 128;       // 2 KB, 128-byte swizzled
constexpr int kStageBytes = kStageA + kStageX;
constexpr int kStages = 2;               // per CTA; kDecodeCtasPerSm CTAs share an SM
constexpr int kSmemData = kStages * kStageBytes;
constexpr int kSmemBytes = kSmemData + 1024 + 256;
constexpr int kECol = 2 * kBN;           // metadata columns after the two accumulators
constexpr int kTmemCols = 64;

// Named barrier of one epilogue warpgroup (id 1 + its index).
__device__ __forceinline__ void epi_bar(int g) { asm volatile("bar.sync %0, 128;" ::"r"(g + 1) : "memory"); }

__global__ void __launch_bounds__(kThreads, kDecodeCtasPerSm)
    hybrid_decode_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
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
    volatile int* last_flag = abort_flag + 1;  // one per epilogue warpgroup

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

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
        b0 = 2 * (int)(((int64_t)p * L.KC) / L.P);
        b1 = min(L.KB, 2 * (int)(((int64_t)(p + 1) * L.KC) / L.P));
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
                const int s = lu / L.P, p = lu % L.P;
                int b0, b1;
                part_range(L, p, b0, b1);
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const uint32_t* mrow = L.meta + (size_t)s * L.KC;
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
                    mbar_arrive_expect_tx(&full[stage], bytes_a + (first ? kMetaBytes : 0) + kStageX);
                    // the packed bytes viewed as 128-byte rows: one 2-D box per record
                    tma_load_2d(st, sp ? &maps.a8[l] : &maps.a16[l], &full[stage], 0, (int)(slab_offset_bytes(d) >> 7));
                    if (first)
                        tma_load_2d(st + kSparseValBytes, &maps.e[l], &full[stage], 0, (int)(mrow[b >> 1] >> 3));
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
            const uint32_t idesc_d = idesc_bf16(128, kBN, false);
            const uint32_t idesc_s = idesc_bf16(128, kBN, true);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any_mma = false;
            bool ready = false;  // full[stage] already seen complete by the look-ahead
            int t = 0;
            for (int it = w_begin; it < w_end && ok; ++it, ++t) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int s = lu / L.P, p = lu % L.P;
                int b0, b1;
                part_range(L, p, b0, b1);
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const int acc = t & 1;
                if (!mbar_wait(&acc_empty[acc], ((t >> 1) & 1) ^ 1u, abort_flag)) {
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
        // ---------------- epilogue: warpgroup g (warps 2+4g .. 5+4g) drains every kEpiGroups-th unit ----------------
        const int g = (warp - 2) >> 2;
        const int q = warp & 3;          // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;
        const int leader = 64 + 128 * g;  // first thread of the warpgroup
        int t = 0;
        for (int it = w_begin; it < w_end; ++it, ++t) {
            if (t % kEpiGroups != g) continue;  // another warpgroup's unit
            const int acc = t & 1;
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const LinDesc& L = a.lins[l];
            const int P = L.P;
            const int s = lu / P, p = lu % P;
            if (!mbar_wait(&acc_full[acc], (t >> 1) & 1, abort_flag)) {
                if (lane == 0) raise();
                break;
            }
            tc_fence_after();
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN), v);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            __nv_bfloat16* yc = a.Y[l] + (size_t)s * kStrip + row;
            if (P == 1) {
                // whole strip in one unit: no partial sums
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                    if (c < a.M) yc[(size_t)c * L.N] = __float2bfloat16_rn(__uint_as_float(v[c]));
                continue;
            }
            // this unit's partial: workspace[s][p][row][0..15]
            float4* dst = reinterpret_cast<float4*>(a.partial[l] + (((size_t)s * P + p) * 128 + row) * kBN);
#pragma unroll
            for (int c = 0; c < kBN / 4; ++c)
                dst[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                     __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
            epi_bar(g);
            if ((int)threadIdx.x == leader) {
                // the barrier orders the warpgroup's stores before this fence,
                // which releases them with the arrival
                __threadfence();
                const unsigned old = atomicAdd(&a.counters[l][s], 1u);
                last_flag[g] = (old == (unsigned)(P - 1));
            }
            epi_bar(g);
            if (last_flag[g]) {
                __threadfence();
                float sum[kBN];
#pragma unroll
                for (int c = 0; c < kBN; ++c) sum[c] = 0.f;
                for (int pp = 0; pp < P; ++pp) {
                    const float4* src =
                        reinterpret_cast<const float4*>(a.partial[l] + (((size_t)s * P + pp) * 128 + row) * kBN);
#pragma unroll
                    for (int c = 0; c < kBN / 4; ++c) {
                        const float4 f = __ldcg(src + c);
                        sum[4 * c] += f.x;
                        sum[4 * c + 1] += f.y;
                        sum[4 * c + 2] += f.z;
                        sum[4 * c + 3] += f.w;
                    }
                }
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                    if (c < a.M) yc[(size_t)c * L.N] = __float2bfloat16_rn(sum[c]);
                if ((int)threadIdx.x == leader) a.counters[l][s] = 0u;  // re-armed for the next call
            }
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

cudaError_t decode_prepare() {
    return cudaFuncSetAttribute(hybrid_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

cudaError_t launch_decode(const GroupMaps& maps, const GroupArgs& a, int grid, cudaStream_t st) {
    hybrid_decode_kernel<<<grid, kThreads, kSmemBytes, st>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace patch
