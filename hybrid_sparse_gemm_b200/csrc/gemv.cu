// Decode-sized product (M <= 16 tokens) on CUDA cores, straight from the
// packed slabs.
//
// At decode sizes the layer is bound by the bytes of W it must stream, and
// the compressed 2:4 slabs carry 1.125 bytes per weight instead of 2
// (PATCH's speedup claim for its hybrid kernel, abstract of "PATCH:
// Learnable Tile-level Hybrid Sparsity for LLMs"). One CTA owns 16 rows of a
// strip; its 8 warps take every 8th slab along K; lane (rg, L) covers rows
// rg, rg+4, rg+8, rg+12 and the 8 columns 8L..8L+7 of each slab, so the X
// slice it needs is the same for dense and sparse slabs and is reused over
// four rows. Partial sums meet in shared memory in a fixed order.
#include "kernels.cuh"

namespace patch {

namespace {

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ float sel4(float x0, float x1, float x2, float x3, uint32_t i) {
    const float lo = (i & 1u) ? x1 : x0;
    const float hi = (i & 1u) ? x3 : x2;
    return (i & 2u) ? hi : lo;
}

template <int MT>
__global__ void __launch_bounds__(256) hybrid_gemv_kernel(const GemvArgs a) {
    const int s = blockIdx.x >> 3, h = blockIdx.x & 7;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = lane & 7, rg = lane >> 3;
    const uint32_t* trow = a.slab + (size_t)s * a.KB;
    const uint32_t* mrow = a.meta + (size_t)s * a.KC;

    float acc[4][MT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[i][m] = 0.f;

    for (int b = warp; b < a.KB; b += 8) {
        const uint32_t d = __ldg(trow + b);
        const uint8_t* base = a.packed + slab_offset_bytes(d);
        float x[MT][8];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m < a.M) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + b * kSlabK + 8 * L));
                x[m][0] = bf_lo(xv.x); x[m][1] = bf_hi(xv.x);
                x[m][2] = bf_lo(xv.y); x[m][3] = bf_hi(xv.y);
                x[m][4] = bf_lo(xv.z); x[m][5] = bf_hi(xv.z);
                x[m][6] = bf_lo(xv.w); x[m][7] = bf_hi(xv.w);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[m][e] = 0.f;
            }
        }
        if (!(d & kSlabSparse)) {
            uint4 wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * h + rg + 4 * i;
                wv[i] = __ldg(reinterpret_cast<const uint4*>(base + sw128_off(r, L)));
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t u[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const float w0 = bf_lo(u[e2]), w1 = bf_hi(u[e2]);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        acc[i][m] = fmaf(w0, x[m][2 * e2], acc[i][m]);
                        acc[i][m] = fmaf(w1, x[m][2 * e2 + 1], acc[i][m]);
                    }
                }
            }
        } else {
            const uint8_t* meta = a.packed + (uint64_t)__ldg(mrow + (b >> 1)) * 16;
            const int kc = (b & 1) * kSlabK + 8 * L;
            uint2 cv[4];
            uint32_t code8[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * h + rg + 4 * i;
                cv[i] = __ldg(reinterpret_cast<const uint2*>(base + sw64_off(r, L >> 1) + (L & 1) * 8));
                code8[i] = __ldg(meta + meta_lane(r, kc) * 16 + (kc >> 5) * 4 + (meta_bit(r, kc) >> 3));
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t u[2] = {cv[i].x, cv[i].y};
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const uint32_t code = (code8[i] >> (4 * g)) & 15u;
                    const uint32_t i0 = code & 3u, i1 = code >> 2;
                    const float v0 = bf_lo(u[g]), v1 = bf_hi(u[g]);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float* xg = &x[m][4 * g];
                        acc[i][m] = fmaf(v0, sel4(xg[0], xg[1], xg[2], xg[3], i0), acc[i][m]);
                        acc[i][m] = fmaf(v1, sel4(xg[0], xg[1], xg[2], xg[3], i1), acc[i][m]);
                    }
                }
            }
        }
    }

    // lanes with the same rg hold the same rows: reduce over L
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = acc[i][m];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            acc[i][m] = v;
        }
    __shared__ float red[8][16][MT];
    if (L == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < MT; ++m) red[warp][rg + 4 * i][m] = acc[i][m];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < 16 * MT; t += blockDim.x) {
        const int row = t / MT, m = t % MT;
        if (m < a.M) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) sum += red[w][row][m];
            a.Y[(size_t)m * a.N + (size_t)s * kStrip + 16 * h + row] = __float2bfloat16_rn(sum);
        }
    }
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st) {
    const int grid = (a.N / kStrip) * 8;
    if (a.M <= 1)
        hybrid_gemv_kernel<1><<<grid, 256, 0, st>>>(a);
    else if (a.M <= 2)
        hybrid_gemv_kernel<2><<<grid, 256, 0, st>>>(a);
    else if (a.M <= 4)
        hybrid_gemv_kernel<4><<<grid, 256, 0, st>>>(a);
    else if (a.M <= 8)
        hybrid_gemv_kernel<8><<<grid, 256, 0, st>>>(a);
    else if (a.M <= 16)
        hybrid_gemv_kernel<16><<<grid, 256, 0, st>>>(a);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace patch
