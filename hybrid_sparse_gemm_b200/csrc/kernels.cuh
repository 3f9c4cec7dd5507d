// Kernel argument structs and launch entry points shared by the host runtime.
#pragma once

#include "common.cuh"

namespace patch {

struct PackArgs {
    const uint16_t* W;        // N x K bf16 bits, row-major
    const uint8_t* bits;      // bit-packed keep mask
    int bitorder;             // 0 MSB first, 1 LSB first
    const uint8_t* flags;     // tile flags on the device, (N/R) x (K/C)
    const uint32_t* table;    // slab table, S x KB
    uint8_t* out;             // packed bytes
    int64_t K;
    int R, C, KB;
    unsigned long long* counters;  // [bad groups, stray zeros, pruned]
};

__global__ void pack_kernel(const PackArgs a);
__global__ void unpack_kernel(const uint8_t* __restrict__ packed, const uint32_t* __restrict__ table,
                              int KB, int64_t K, uint16_t* __restrict__ Wm);

struct GemmArgs {
    const uint8_t* packed;
    const uint32_t* table;   // S x KB slab table
    const int* work_off;     // per CTA: [work_off[c], work_off[c+1]) into work
    const int* work;         // unit = strip * MB + m_block
    int M, N, KB, MB;
    __nv_bfloat16* Y;
    int* status;             // device status word (timeouts)
};

struct GemvArgs {
    const uint8_t* packed;
    const uint32_t* table;
    const __nv_bfloat16* X;  // M x K
    __nv_bfloat16* Y;        // M x N
    int M, N, K, KB;
};

// Launchers (return cudaError_t of the launch).
cudaError_t launch_gemm(const CUtensorMap& tmap_x, const GemmArgs& a, int grid, int bn, cudaStream_t st);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);
int gemm_bn_for(int M);
cudaError_t gemm_prepare();  // one-time function attributes

}  // namespace patch
