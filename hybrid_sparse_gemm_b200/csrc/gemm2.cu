// Hybrid dense / 2:4 GEMM on CTA pairs (cta_group::2): Y = X . (W (.) Mask)^T.
//
// Same method as the single-CTA kernel (dense slabs on tcgen05.mma, 2:4 slabs
// on tcgen05.mma.sp; PATCH abstract, "PATCH: Learnable Tile-level Hybrid
// Sparsity for LLMs"), on the unit Blackwell's tensor core is built around:
// two CTAs on neighbouring SMs form one 256 x 256 MMA. CTA r of a pair holds
// the 128 weight rows of one strip (operand A) and tokens [128r, 128r+128) of
// the block (operand B); each MMA multiplies both A halves by both B halves,
// so an SM loads half the activations it would need alone. The pair's leader
// (even rank) issues every MMA; both CTAs' TMA loads complete on the leader's
// barriers, and the leader's commits arrive on the CTAs' barriers.
//
// With CL = 4 two pairs (four strips) share a cluster and a token block: each
// activation sub-tile is loaded once and multicast to the CTA of each pair
// that needs it, halving the activation bytes each SM pulls from L2. The two
// pairs then advance through the shared stages together (a stage is free
// when both pairs' MMAs have consumed it).
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

namespace patch {

namespace {

constexpr int kThreads = 192;
constexpr int kHalf = 128;                    // tokens per CTA
constexpr int kStages = 6;
constexpr int kStageA = 18432;                // 16 KB dense, or 8 KB values + 2 KB metadata
constexpr int kStageB = kHalf * 128;          // 16 KB
constexpr int kSmemData = kStages * (kStageA + kStageB);
constexpr int kSmemBytes = kSmemData + 1024 + 256;
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kETail = kAccCols - 4;          // metadata columns inside the idle accumulator
constexpr uint32_t kPeerMask = 0xFEFFFFFFu;   // clears the CTA-in-pair bit of a shared address

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 2-D TMA load whose completion is counted on the pair leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
// The same load written to the same offset in every CTA of `mask`; each
// destination's bytes complete on its own pair leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair_mc(uint32_t dst, const CUtensorMap* map, uint32_t bar_local,
                                                    int c0, int c1, uint16_t mask) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.multicast::cluster"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(map), "r"(bar_local & kPeerMask), "r"(c0), "r"(c1), "h"(mask)
        : "memory");
}
__device__ __forceinline__ void mma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma2_sp_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t e_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%5], %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e_tmem)
        : "memory");
}
__device__ __forceinline__ void cp2_128x128b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// Commit of the leader's MMAs, arriving on the barrier at this offset in every
// CTA of `mask`.
__device__ __forceinline__ void commit2_mask(uint64_t* bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(mask)
        : "memory");
}
__device__ __forceinline__ void commit2_local(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

template <int CL>
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_gemm2_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
    constexpr int kStrips = CL;            // strips per cluster (one per CTA)
    constexpr int kPairs = CL / 2;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kStageA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
    uint64_t* full = bars;                    // pair leader: both CTAs' bytes of a stage
    uint64_t* empty = bars + kStages;         // every CTA: stage consumed by every pair's MMAs
    uint64_t* acc_full = bars + 2 * kStages;  // both CTAs of a pair: accumulator ready
    uint64_t* acc_empty = acc_full + 2;       // pair leader: 8 epilogue warps drained it
    uint64_t* e_free = acc_full + 4;          // pair leader: 8 epilogue warps read its tail
    uint64_t* drain = acc_full + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t pr = rank & 1u;          // CTA within its pair
    const uint32_t pair = rank >> 1;        // pair within the cluster
    const uint32_t leader = rank & ~1u;
    const uint16_t pair_mask = (uint16_t)(3u << leader);
    const uint16_t all_mask = (uint16_t)((1u << CL) - 1u);
    const int cl = blockIdx.x / CL;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kPairs);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);
            mbar_init(&e_free[i], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
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
    // strip this CTA loads for cluster-unit c of a member with S strips
    auto own_strip = [&](int c, int S) {
        int s = kStrips * c + (int)rank;
        if (s >= S) s = kStrips * c + (int)pr;
        if (s >= S) s = kStrips * c;
        return s;
    };

    const int w_begin = a.work_off[cl];
    const int w_end = a.work_off[cl + 1];

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer (every CTA) ----------------
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int it = w_begin; it < w_end && ok; ++it) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int c = lu / a.MB, j = lu % a.MB;
                const int s = own_strip(c, L.S);
                const uint32_t* trow = L.gemm + (size_t)s * L.KB;
                const uint32_t* mrow = L.meta + (size_t)s * L.KC;
                const int KB = L.KB;
                const CUtensorMap* tm_x = &maps.x[l];
                const CUtensorMap* tm_a16 = &maps.a16[l];
                const CUtensorMap* tm_a8 = &maps.a8[l];
                const CUtensorMap* tm_e = &maps.e[l];
                for (int b = 0; b < KB; ++b) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    const uint32_t d = trow[b];
                    const bool sp = d & kSlabSparse, first = d & kSlabFirst;
                    const uint32_t bar = map_to_rank(smem_u32(&full[stage]), leader);
                    if (pr == 0)
                        mbar_arrive_expect_tx(&full[stage],
                                              2u * ((sp ? kSparseValBytes : kDenseSlabBytes) +
                                                    (first ? kMetaBytes : 0) + kStageB));
                    const uint32_t dst_a = smem_u32(sA + stage * kStageA);
                    const int row = (int)(slab_offset_bytes(d) >> 7);
                    tma_load_2d_pair(dst_a, sp ? tm_a8 : tm_a16, bar, 0, row);
                    if (first)
                        tma_load_2d_pair(dst_a + kSparseValBytes, tm_e, bar, 0, (int)(mrow[b >> 1] >> 3));
                    const int tok = j * kGemm2BN + (int)pr * kHalf;
                    if (CL == 2) {
                        tma_load_2d_pair(smem_u32(sB + stage * kStageB), tm_x, bar, b * kSlabK, tok);
                    } else {
                        // this CTA fetches half of its 128 activation rows and
                        // multicasts them to the same CTA of the other pair
                        const uint32_t off = pair * (kStageB / 2);
                        tma_load_2d_pair_mc(smem_u32(sB + stage * kStageB) + off, tm_x, smem_u32(&full[stage]),
                                            b * kSlabK, tok + (int)pair * (kHalf / 2),
                                            (uint16_t)((1u << pr) | (1u << (pr + 2))));
                    }
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (pr == 0) {
                // Bounded wait for the loads of the last stages, whatever the
                // abort flag says, so none lands after the cluster exits.
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
        }
    } else if (warp == 1) {
        if (lane == 0 && pr == 0) {
            // ---------------- MMA issuer (pair leader) ----------------
            const uint32_t idesc_d = idesc_bf16(256, kGemm2BN, false);
            const uint32_t idesc_s = idesc_bf16(256, kGemm2BN, true);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any_mma = false;
            int t = 0;
            for (int it = w_begin; it < w_end && ok; ++it, ++t) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int c = lu / a.MB;
                const uint32_t* trow = L.gemm + (size_t)own_strip(c, L.S) * L.KB;
                const int KB = L.KB;
                const int acc = t & 1;
                if (!mbar_wait(&acc_empty[acc], ((t >> 1) & 1) ^ 1u, abort_flag)) {
                    raise();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
                const uint32_t e_base = tmem_base + (uint32_t)((1 - acc) * kAccCols + kETail);
                bool e_ready = (t == 0);
                for (int b = 0; b < KB; ++b) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        raise();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = trow[b];
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
                    commit2_mask(&empty[stage], all_mask);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                commit2_mask(&acc_full[acc], pair_mask);
            }
            if (*abort_flag && any_mma) {
                commit2_local(drain);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5, every CTA) ----------------
        const int q = warp & 3;
        int t = 0;
        for (int it = w_begin; it < w_end; ++it, ++t) {
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const int N = a.lins[l].N;
            const int c = lu / a.MB, j = lu % a.MB;
            const int s = kStrips * c + (int)rank;
            const bool store = s < a.lins[l].S;
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
                    if (lane == 0) remote_arrive(map_to_rank(smem_u32(&e_free[acc]), leader));
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
            if (lane == 0) remote_arrive(map_to_rank(smem_u32(&acc_empty[acc]), leader));
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while another may still signal it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc2(tmem_base, kTmemCols);
    }
}

template <int CL>
cudaError_t prepare(int* max_clusters) {
    cudaError_t e =
        cudaFuncSetAttribute(hybrid_gemm2_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = CL;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, hybrid_gemm2_kernel<CL>, &cfg);
    if (e != cudaSuccess) return e;
    *max_clusters = n;
    return cudaSuccess;
}

template <int CL>
cudaError_t launch(const GroupMaps& maps, const GroupArgs& a, int clusters, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = CL;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, hybrid_gemm2_kernel<CL>, maps, a);
}

}  // namespace

cudaError_t gemm_prepare_pair(int* max_pair_clusters, int* max_quad_clusters) {
    cudaError_t e = prepare<2>(max_pair_clusters);
    if (e != cudaSuccess) return e;
    return prepare<4>(max_quad_clusters);
}

cudaError_t launch_gemm2(const GroupMaps& maps, const GroupArgs& a, int clusters, int cluster_ctas, cudaStream_t st) {
    return cluster_ctas == 4 ? launch<4>(maps, a, clusters, st) : launch<2>(maps, a, clusters, st);
}

}  // namespace patch
