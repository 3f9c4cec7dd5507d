// Hybrid dense / 2:4 GEMM on sm_100a: Y = X . (W (.) Mask)^T.
//
// PATCH's speed comes from a kernel that runs dense tiles on the dense tensor
// core path and 2:4 tiles on the structured-sparse one (abstract of "PATCH:
// Learnable Tile-level Hybrid Sparsity for LLMs"; "How to use" on the
// "llama_3.2_1b-PATCH-45Sparse" card). This kernel is written for Blackwell:
//
//  * swap-AB: the weight is the MMA's A operand (M_mma = 128 weight rows, the
//    only operand the sparse MMA can compress) and the activations are B
//    (N_mma = BN tokens); the accumulator is a 128 x BN fp32 tile of Y^T in
//    tensor memory.
//  * one persistent CTA per SM walks a cost-balanced list of output tiles
//    (strip of 128 weight rows, block of BN tokens);
//  * warp 0 streams each 64-column slab: the packed weight slab (already in the
//    tensor core's shared-memory image) by one bulk copy, the X tile by a 2-D
//    TMA load with 128-byte swizzle;
//  * warp 1 issues tcgen05.mma (dense slab: 4 x K16) or tcgen05.mma.sp
//    (sparse slab: 2 x K32, metadata moved to TMEM by tcgen05.cp) into one of
//    two TMEM accumulators, and commits each stage back to the producer;
//  * warps 2..5 drain the other accumulator (tcgen05.ld, fp32 -> bf16) while
//    the next tile accumulates.
// Every wait is bounded: on expiry the CTA records a timeout in the status
// word, drains its own copies and MMAs, frees TMEM and returns.
#include "kernels.cuh"

namespace patch {

namespace {

constexpr int kThreads = 192;
constexpr int kStageABytes = 18432;  // 16 KB dense, or 8 KB values + 2 KB metadata

template <int BN>
struct Cfg {
    static constexpr int kStageBBytes = BN * 128;
    static constexpr int kStages = (BN >= 128) ? 6 : 8;
    static constexpr int kECol = 2 * BN;  // 4 metadata columns after the accumulators
    static constexpr int kTmemCols = (2 * BN + 4 <= 32) ? 32 : (2 * BN + 4 <= 64) ? 64
                                   : (2 * BN + 4 <= 128) ? 128 : (2 * BN + 4 <= 256) ? 256 : 512;
    static constexpr int kSmemData = kStages * (kStageABytes + kStageBBytes);
    static constexpr int kSmemBytes = kSmemData + 1024 /*align*/ + 256 /*barriers*/;
};

struct Abort {
    int* status;
    volatile int* flag;
    __device__ void raise() const {
        *flag = 1;
        atomicCAS(status, 0, kStatusTimeout);
    }
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_gemm_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs a) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::kStages * kStageABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemData);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* acc_full = bars + 2 * C::kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_full + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const Abort ab{a.status, abort_flag};

    const int w_begin = a.work_off[blockIdx.x];
    const int w_end = a.work_off[blockIdx.x + 1];

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
                const int s = lu / a.MB, j = lu % a.MB;
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const uint32_t* mrow = L.meta + (size_t)s * L.KC;
                const CUtensorMap* tmap_x = &maps.x[l];
                const int KB = L.KB;
                uint32_t d_next = trow[0];
                for (int b = 0; b < KB; ++b) {
                    const uint32_t d = d_next;
                    if (b + 1 < KB) d_next = trow[b + 1];  // fetched one slab ahead
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ab.raise();
                        ok = false;
                        break;
                    }
                    const bool sp = d & kSlabSparse, first = d & kSlabFirst;
                    const uint32_t bytes_a = sp ? kSparseValBytes : kDenseSlabBytes;
                    mbar_arrive_expect_tx(&full[stage], bytes_a + (first ? kMetaBytes : 0) + C::kStageBBytes);
                    // the packed bytes viewed as 128-byte rows: one 2-D box per record
                    tma_load_2d(sA + stage * kStageABytes, sp ? &maps.a8[l] : &maps.a16[l], &full[stage], 0,
                                (int)(slab_offset_bytes(d) >> 7));
                    if (first)
                        tma_load_2d(sA + stage * kStageABytes + kSparseValBytes, &maps.e[l], &full[stage], 0,
                                    (int)(mrow[b >> 1] >> 3));
                    tma_load_2d(sB + stage * C::kStageBBytes, tmap_x, &full[stage], b * kSlabK, j * BN);
                    ++issued;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Wait (bounded, whatever the abort flag says) for the copies still
            // in flight so none lands after this CTA exits.
            int st = stage;
            uint32_t ph = phase;
            for (int i = 0; i < C::kStages && i < issued; ++i) {
                if (--st < 0) {
                    st = C::kStages - 1;
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
            const uint32_t idesc_d = idesc_bf16(128, BN, false);
            const uint32_t idesc_s = idesc_bf16(128, BN, true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            bool any_mma = false;
            bool ready = false;  // full[stage] already seen complete by the look-ahead
            for (int it = w_begin; it < w_end && ok; ++it) {
                const int u = a.work[it];
                const int l = u >> kUnitShift, lu = u & kUnitMask;
                const LinDesc& L = a.lins[l];
                const int s = lu / a.MB;
                const uint32_t* trow = L.slab + (size_t)s * L.KB;
                const int KB = L.KB;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    ab.raise();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                uint32_t d = trow[0];
                for (int b = 0; b < KB; ++b) {
                    // the record comes one slab ahead and the next stage is
                    // tested before this slab's MMAs (see the pair kernel)
                    if (!ready && !mbar_wait(&full[stage], phase, abort_flag)) {
                        ab.raise();
                        ok = false;
                        break;
                    }
                    const uint32_t d_next = b + 1 < KB ? trow[b + 1] : 0u;
                    int next = stage + 1;
                    uint32_t next_phase = phase;
                    if (next == C::kStages) {
                        next = 0;
                        next_phase ^= 1u;
                    }
                    ready = mbar_test_wait(&full[next], next_phase);
                    const uint32_t a_addr = smem_u32(sA + stage * kStageABytes);
                    const uint32_t b_addr = smem_u32(sB + stage * C::kStageBBytes);
                    if (d & kSlabSparse) {
                        if (d & kSlabFirst)
                            tc_cp_128x128b(tmem_base + C::kECol,
                                           smem_desc(a_addr + kSparseValBytes, 16, 128, kLayoutNone));
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 512, kLayoutSw64);
                            const uint64_t bd = smem_desc(b_addr + i * 64, 16, 1024, kLayoutSw128);
                            const uint32_t ecol = C::kECol + (b & 1) * 2 + i;
                            mma_sp_bf16(d_tmem, ad, bd, idesc_s | (ecol & 1u), tmem_base + (ecol & ~1u),
                                        (b | i) != 0);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint64_t ad = smem_desc(a_addr + i * 32, 16, 1024, kLayoutSw128);
                            const uint64_t bd = smem_desc(b_addr + i * 32, 16, 1024, kLayoutSw128);
                            mma_bf16(d_tmem, ad, bd, idesc_d, (b | i) != 0);
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
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (*abort_flag && any_mma) {
                // Let issued MMAs finish before TMEM is released.
                tc_commit(drain);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int it = w_begin; it < w_end; ++it) {
            const int u = a.work[it];
            const int l = u >> kUnitShift, lu = u & kUnitMask;
            const int N = a.lins[l].N;
            const int s = lu / a.MB, j = lu % a.MB;
            if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag)) {
                if (lane == 0) ab.raise();
                break;
            }
            tc_fence_after();
            const int n = s * kStrip + q * 32 + lane;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            __nv_bfloat16* yc = a.Y[l] + n;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + c0, v);
                tc_wait_ld();
                const int m0 = j * BN + c0;
                if (m0 + 32 <= a.M) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        yc[(size_t)(m0 + c) * N] = __float2bfloat16_rn(__uint_as_float(v[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (m0 + c < a.M)
                            yc[(size_t)(m0 + c) * N] = __float2bfloat16_rn(__uint_as_float(v[c]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int BN>
cudaError_t set_attr() {
    return cudaFuncSetAttribute(hybrid_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<BN>::kSmemBytes);
}

}  // namespace

cudaError_t gemm_prepare_single() { return set_attr<kGemmBN>(); }

cudaError_t launch_gemm(const GroupMaps& maps, const GroupArgs& a, int grid, cudaStream_t st) {
    hybrid_gemm_kernel<kGemmBN><<<grid, kThreads, Cfg<kGemmBN>::kSmemBytes, st>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace patch
