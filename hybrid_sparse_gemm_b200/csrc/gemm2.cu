// Hybrid dense / 2:4 GEMM on CTA pairs (cta_group::2): Y = X . (W (.) Mask)^T.
//
// Same method as the single-CTA kernel (dense slabs on tcgen05.mma, 2:4 slabs
// on tcgen05.mma.sp; PATCH abstract, "PATCH: Learnable Tile-level Hybrid
// Sparsity for LLMs"), on the unit Blackwell's tensor core is built around:
// two CTAs on neighbouring SMs form one 256 x 256 MMA. CTA r of a pair holds
// the 128 weight rows of one strip (operand A) and tokens [128r, 128r+128) of
// the block (operand B); each MMA multiplies both A halves by both B halves,
// so an SM loads half the activations it would need alone. The pair's leader
// (rank 0) issues every MMA; both CTAs' TMA loads complete on the leader's
// barriers, and the leader's commits arrive on the CTAs' barriers.
//
// TMEM: each CTA holds its 128 rows x 256 tokens in one of two 256-column
// accumulators. The 2:4 metadata of the running tile lives in the last four
// columns of the other accumulator: its epilogue drains those columns first
// and releases them early (e_free) so the next tile's tcgen05.cp can land.
//
// Both strips of a pair load the same kind of record at every slab (dense
// images stand in for 2:4 slabs whose partner is dense), so one MMA
// instruction always covers both. Strips past the end of the weight (an odd
// last strip, a last cluster with fewer strips) are replaced by duplicates
// whose results are not stored.
#include "kernels.cuh"
#include "pair.cuh"

namespace patch {

namespace {

#ifndef PATCH_GEMM2_PRODUCERS
#define PATCH_GEMM2_PRODUCERS 2
#endif
constexpr int kProducers = PATCH_GEMM2_PRODUCERS;  // TMA-issuing warps per CTA (slabs dealt round robin)
constexpr int kMmaWarp = kProducers;              // MMA issuer (pair leader) and TMEM owner
constexpr int kThreads = 32 * (kProducers + 1 + 4);
constexpr int kHalf = 128;                    // tokens per CTA
constexpr int kStages = 6;
static_assert(kStages % 2 == 0 && kStages % kProducers == 0, "stages come in pairs dealt round robin");
constexpr int kStageA = 18432;                // 16 KB dense, or 8 KB values + 2 KB metadata
constexpr int kStageB = kHalf * 128;          // 16 KB
constexpr int kSmemData = kStages * (kStageA + kStageB);
constexpr int kSmemBytes = kSmemData + 1024 + 256;
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kETail = kAccCols - 4;          // metadata columns inside the idle accumulator
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_gemm2_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kStageA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
    uint64_t* full = bars;                       // pair leader: both CTAs' bytes of a stage
    uint64_t* empty = bars + kStages;            // both CTAs: a stage pair consumed by the MMAs
    uint64_t* acc_full = empty + kStages / 2;    // both CTAs of a pair: accumulator ready
    uint64_t* acc_empty = acc_full + 2;          // pair leader: 8 epilogue warps drained it
    uint64_t* e_free = acc_full + 4;             // pair leader: 8 epilogue warps read its tail
    uint64_t* drain = acc_full + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t pr = cluster_rank();     // CTA within the pair (0 = leader)
    const int cl = blockIdx.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
        for (int i = 0; i < kStages / 2; ++i) mbar_init(&empty[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);
            mbar_init(&e_free[i], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc2(tmem_slot, kTmemCols);
        tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers of every CTA initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto raise = [&]() {
        *abort_flag = 1;
        atomicCAS(a.status, 0, kStatusTimeout);
    };
    // pair position of the strip this CTA loads for pair-unit c of member L
    // (an odd last strip is duplicated into the second CTA and not stored);
    // the tables L.gemm and L.pmeta have their rows in this order
    auto own_pos = [&](const LinDesc& L, int c) {
        const int pos = 2 * c + (int)pr;
        return pos < L.S ? pos : 2 * c;
    };

    const int w_begin = a.work_off[cl];
    const int w_end = a.work_off[cl + 1];

    if (warp < kProducers) {
        if (lane == 0) {
            // ---------------- producers (every CTA) ----------------
            // Slab g of this CTA's sequence goes to stage g % kStages and is
            // loaded by producer g % kProducers; a stage pair (2q, 2q+1) is
            // released by one commit after the MMAs of its second slab.
            const int me = warp;
            int g0 = 0;           // sequence index of the current unit's first slab
            int my_last = -1;     // sequence index of the last slab this producer loaded
            bool ok = true;
            for (int it = w_begin; it < w_end && ok; ++it) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int c = lu / a.MB, j = lu % a.MB;
                const int pos = own_pos(L, c);
                const uint32_t* trow = L.gemm + (size_t)pos * L.KB;
                const uint32_t* mrow = L.pmeta + (size_t)pos * L.KC;
                const int KB = L.KB;
                const CUtensorMap* tm_x = &maps.x[l];
                const CUtensorMap* tm_a16 = &maps.a16[l];
                const CUtensorMap* tm_a8 = &maps.a8[l];
                const CUtensorMap* tm_e = &maps.e[l];
                const int tok = j * kGemm2BN + (int)pr * kHalf;
                // slab b of this unit is slab g0 + b of the CTA's sequence
                int b = ((me - g0) % kProducers + kProducers) % kProducers;
                uint32_t d_next = b < KB ? trow[b] : 0u;
                for (; b < KB; b += kProducers) {
                    const uint32_t d = d_next;
                    if (b + kProducers < KB) d_next = trow[b + kProducers];  // fetched one slab ahead
                    const int g = g0 + b;
                    const int q = g >> 1;
                    if (!mbar_wait(&empty[q % (kStages / 2)], ((q / (kStages / 2)) & 1) ^ 1u, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const int stage = g % kStages;
                    const bool sp = d & kSlabSparse, first = d & kSlabFirst;
                    const uint32_t bar = map_to_rank(smem_u32(&full[stage]), 0);
                    if (pr == 0)
                        mbar_arrive_expect_tx(&full[stage],
                                              2u * ((sp ? kSparseValBytes : kDenseSlabBytes) +
                                                    (first ? kMetaBytes : 0) + kStageB));
                    const uint32_t dst_a = smem_u32(sA + stage * kStageA);
                    tma_load_2d_pair(dst_a, sp ? tm_a8 : tm_a16, bar, 0, (int)(slab_offset_bytes(d) >> 7));
                    if (first)
                        tma_load_2d_pair(dst_a + kSparseValBytes, tm_e, bar, 0, (int)(mrow[b >> 1] >> 3));
                    tma_load_2d_pair(smem_u32(sB + stage * kStageB), tm_x, bar, b * kSlabK, tok);
                    my_last = g;
                }
                g0 += KB;
            }
            if (pr == 0) {
                // Bounded wait for the loads of my last stages, whatever the
                // abort flag says, so none lands after the cluster exits.
                for (int g = my_last - kStages + 1; g <= my_last; ++g) {
                    if (g < 0 || g % kProducers != me) continue;
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&full[g % kStages], (uint32_t)((g / kStages) & 1)) &&
                           globaltimer() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0 && pr == 0) {
            // ---------------- MMA issuer (pair leader) ----------------
            const uint32_t idesc_d = idesc_bf16(256, kGemm2BN, false);
            const uint32_t idesc_s = idesc_bf16(256, kGemm2BN, true);
            int stage = 0;
            uint32_t phase = 0;
            int g = 0;
            bool ok = true, any_mma = false;
            bool ready = false;  // full[stage] already seen complete by the look-ahead
            int t = 0;
            for (int it = w_begin; it < w_end && ok; ++it, ++t) {
                const int u = a.work[it];
                const LinDesc& L = a.lins[u >> kUnitShift];
                const int KB = L.KB;
                const uint32_t* trow = L.gemm + (size_t)own_pos(L, (u & kUnitMask) / a.MB) * KB;
                uint32_t d = trow[0];
                const int acc = t & 1;
                if (!mbar_wait(&acc_empty[acc], ((t >> 1) & 1) ^ 1u, abort_flag)) {
                    raise();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
                const uint32_t e_base = tmem_base + (uint32_t)((1 - acc) * kAccCols + kETail);
                bool e_ready = (t == 0);
                for (int b = 0; b < KB; ++b, ++g) {
                    // Nothing that depends on this slab's data sits between the
                    // wait and the MMAs: the record was fetched one slab ahead,
                    // and the next stage is tested (without blocking) before
                    // this slab's MMAs so that its wait is usually free.
                    if (!ready && !mbar_wait(&full[stage], phase, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const uint32_t d_next = b + 1 < KB ? trow[b + 1] : 0u;
                    int next = stage + 1;
                    uint32_t next_phase = phase;
                    if (next == kStages) {
                        next = 0;
                        next_phase ^= 1u;
                    }
                    ready = mbar_test_wait(&full[next], next_phase);
                    const uint32_t a_addr = smem_u32(sA + stage * kStageA);
                    const uint32_t b_addr = smem_u32(sB + stage * kStageB);
                    if (d & kSlabSparse) {
                        if (d & kSlabFirst) {
                            if (!e_ready) {
                                if (!mbar_wait(&e_free[1 - acc], ((t - 1) >> 1) & 1, abort_flag)) {
                                    raise();
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                e_ready = true;
                            }
                            cp2_128x128b(e_base, smem_desc(a_addr + kSparseValBytes, 16, 128, kLayoutNone));
                        }
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 512, kLayoutSw64);
                            const uint64_t bd = smem_desc(b_addr + i * 64, 16, 1024, kLayoutSw128);
                            const uint32_t ecol = e_base + (uint32_t)((b & 1) * 2 + i);
                            mma2_sp_bf16(d_tmem, ad, bd, idesc_s | (ecol & 1u), ecol & ~1u, (b | i) != 0);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 1024, kLayoutSw128);
                            const uint64_t bd = smem_desc(b_addr + i * 32, 16, 1024, kLayoutSw128);
                            mma2_bf16(d_tmem, ad, bd, idesc_d, (b | i) != 0);
                        }
                    }
                    any_mma = true;
                    if (g & 1) commit2_mask(&empty[(g >> 1) % (kStages / 2)], 3);
                    stage = next;
                    phase = next_phase;
                    d = d_next;
                }
                if (!ok) break;
                commit2_mask(&acc_full[acc], 3);
            }
            if (*abort_flag && any_mma) {
                commit2_local(drain);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---------------- epilogue (4 warps, every CTA) ----------------
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        int t = 0;
        for (int it = w_begin; it < w_end; ++it, ++t) {
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const int N = a.lins[l].N;
            const int c = lu / a.MB, j = lu % a.MB;
            const int pos = 2 * c + (int)pr;  // pair position of this CTA's strip
            const bool store = pos < a.lins[l].S;
            const int s = store ? a.lins[l].order[pos] : 0;
            const int acc = t & 1;
            if (!mbar_wait(&acc_full[acc], (t >> 1) & 1, abort_flag)) {
                if (lane == 0) raise();
                break;
            }
            tc_fence_after();
            const int n = s * kStrip + q * 32 + lane;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols);
            __nv_bfloat16* yc = a.Y[l] + n;
#pragma unroll 1
            for (int c0 = kAccCols - 32; c0 >= 0; c0 -= 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + c0, v);
                tc_wait_ld();
                if (c0 == kAccCols - 32) {
                    // The tail (metadata columns of the next tile) is read: release it.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) remote_arrive(map_to_rank(smem_u32(&e_free[acc]), 0));
                }
                if (!store) continue;
                const int m0 = j * kGemm2BN + c0;
                if (m0 + 32 <= a.M) {
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc)
                        yc[(size_t)(m0 + cc) * N] = __float2bfloat16_rn(__uint_as_float(v[cc]));
                } else {
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc)
                        if (m0 + cc < a.M)
                            yc[(size_t)(m0 + cc) * N] = __float2bfloat16_rn(__uint_as_float(v[cc]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) remote_arrive(map_to_rank(smem_u32(&acc_empty[acc]), 0));
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while another may still signal it
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

cudaError_t gemm_prepare_pair(int* max_clusters) {
    cudaError_t e =
        cudaFuncSetAttribute(hybrid_gemm2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = config(1, &attr, nullptr);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, hybrid_gemm2_kernel, &cfg);
    if (e != cudaSuccess) return e;
    *max_clusters = n;
    return cudaSuccess;
}

cudaError_t launch_gemm2(const GroupMaps& maps, const GroupArgs& a, int clusters, cudaStream_t st) {
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = config(clusters, &attr, st);
    return cudaLaunchKernelEx(&cfg, hybrid_gemm2_kernel, maps, a);
}

}  // namespace patch
