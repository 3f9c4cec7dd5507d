// Kernel argument structs and launch entry points shared by the host runtime.
#pragma once

#include "common.cuh"

namespace patch {

struct PackArgs {
    const uint16_t* W;        // N x K bf16 bits, row-major
    const uint8_t* bits;      // bit-packed keep mask
    int bitorder;             // 0 MSB first, 1 LSB first
    const uint8_t* flags;     // tile flags on the device, (N/R) x (K/C)
    const uint32_t* slab;     // per-strip slab table, S x KB
    const uint32_t* meta;     // metadata block table, S x KC
    const uint32_t* gemm;     // CTA-pair slab table, S x KB
    uint8_t* out;             // packed bytes
    int64_t K;
    int R, C, KB, KC;
    unsigned long long* counters;  // [bad groups, stray zeros, pruned]
};

__global__ void pack_kernel(const PackArgs a);
__global__ void unpack_kernel(const uint8_t* __restrict__ packed, const uint32_t* __restrict__ slab,
                              const uint32_t* __restrict__ meta_tab, int KB, int KC, int64_t K,
                              uint16_t* __restrict__ Wm);

// Tensor-core kernel, one CTA per 128-row strip x 128-token block.
struct GemmArgs {
    const uint8_t* packed;
    const uint32_t* slab;    // per-strip slab table
    const uint32_t* meta;    // metadata block table
    const int* work_off;     // per CTA: [work_off[c], work_off[c+1]) into work
    const int* work;         // unit = strip * MB + m_block
    int M, N, KB, KC, MB;
    __nv_bfloat16* Y;
    int* status;             // device status word (timeouts)
};

// Tensor-core kernel, one CTA pair per 256-row strip pair x 256-token block.
struct Gemm2Args {
    const uint32_t* gemm;    // CTA-pair slab table
    const uint32_t* meta;
    const int* work_off;     // per cluster
    const int* work;         // unit = pair * MB + m_block
    int M, N, S, KB, KC, MB;
    __nv_bfloat16* Y;
    int* status;
};

struct GemvArgs {
    const uint8_t* packed;
    const uint32_t* slab;
    const uint32_t* meta;
    const __nv_bfloat16* X;  // M x K
    __nv_bfloat16* Y;        // M x N
    int M, N, K, KB, KC;
};

// Decode kernel (M <= 16): split-K over persistent CTAs, partials reduced by
// the last CTA of each strip.
struct DecodeArgs {
    const uint8_t* packed;
    const uint32_t* slab;
    const uint32_t* meta;
    const int* work_off;     // per CTA
    const int* work;         // unit = strip * P + part
    int M, N, KB, KC, P;
    float* partial;          // [S][P][128][16] fp32 workspace
    unsigned* counters;      // [S] arrivals per strip, zero between calls
    __nv_bfloat16* Y;
    int* status;
};

// Launchers (return cudaError_t of the launch).
cudaError_t launch_gemm(const CUtensorMap& tmap_x, const GemmArgs& a, int grid, cudaStream_t st);
cudaError_t launch_gemm2(const CUtensorMap& tmap_x, const CUtensorMap& tm_a16, const CUtensorMap& tm_a8,
                         const CUtensorMap& tm_e, const Gemm2Args& a, int clusters, cudaStream_t st);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);
cudaError_t launch_decode(const CUtensorMap& tmap_x, const DecodeArgs& a, int grid, cudaStream_t st);
cudaError_t decode_prepare();
cudaError_t gemm_prepare(int* max_pair_clusters);  // one-time function attributes, cluster occupancy

constexpr int kGemmBN = 128;   // tokens per CTA tile (single-CTA kernel)
constexpr int kGemm2BN = 256;  // tokens per CTA-pair tile
constexpr int kDecodeBN = 16;  // tokens per decode MMA (M <= 16)

}  // namespace patch
