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

// The tensor-core kernels run a group of packed linears (one or more weights
// sharing M, e.g. the projections of one layer) in one persistent launch.
constexpr int kMaxGroup = 8;

// Static description of one packed linear (device memory, built at pack).
struct LinDesc {
    const uint8_t* packed;
    const uint32_t* slab;      // per-strip slab table
    const uint32_t* meta;      // metadata block table
    const uint32_t* gemm;      // CTA-pair slab table, rows in pair-position order
    const uint32_t* pmeta;     // metadata block table, rows in pair-position order
    const int* order;          // strips by pair position: pair i = strips order[2i], order[2i+1]
    int N, S, KB, KC, P;       // P: decode K-parts per strip (16-token instance)
    int PW;                    // decode K-parts per strip of the 64-token instance
};

// Tensor maps: X of every member (per call) and the packed bytes of every
// member viewed as 128-byte rows with 256-, 128-, 64- and 16-row boxes.
struct GroupMaps {
    CUtensorMap x[kMaxGroup];
    CUtensorMap a32[kMaxGroup], a16[kMaxGroup], a8[kMaxGroup], e[kMaxGroup];
};

// Per-call arguments. A work unit is (member << 24) | local index, the local
// index being strip*MB + token block (single-CTA), pair*MB + token block
// (CTA pair) or strip*P + part (decode).
struct GroupArgs {
    const LinDesc* lins;
    __nv_bfloat16* Y[kMaxGroup];
    // decode only: split-K workspace [S][P][BN][128] fp32 and per-strip
    // arrival counters (zero between calls) of each member, owned by the
    // calling stream so that calls on different streams never share them
    float* partial[kMaxGroup];
    unsigned* counters[kMaxGroup];
    const int* work_off;       // per CTA (or per CTA pair): [work_off[c], work_off[c+1])
    const int* work;
    int M, MB;
    // two-strips-per-CTA kernel: its MB token tiles share M's ceil(M/16)
    // 16-token granules, tile_gran each and one more for the first tile_extra
    int tile_gran, tile_extra;
    int* status;               // device status word (timeouts)
};
constexpr int kUnitShift = 24;
constexpr int kUnitMask = (1 << kUnitShift) - 1;

struct GemvArgs {
    const uint8_t* packed;
    const uint32_t* slab;
    const uint32_t* meta;
    const __nv_bfloat16* X;  // M x K
    __nv_bfloat16* Y;        // M x N
    int M, N, K, KB, KC;
};

// Launchers (return cudaError_t of the launch).
cudaError_t launch_gemm(const GroupMaps& maps, const GroupArgs& a, int grid, cudaStream_t st);
cudaError_t launch_gemm2(const GroupMaps& maps, const GroupArgs& a, int clusters, cudaStream_t st);
// pure24: every member's slabs all run on the sparse MMA (no tables read)
cudaError_t launch_gemm22(const GroupMaps& maps, const GroupArgs& a, int clusters, bool pure24, cudaStream_t st);
// bn: tokens per decode MMA, kDecodeBN (M <= 16) or kDecodeWideBN (M <= 64)
cudaError_t launch_decode(const GroupMaps& maps, const GroupArgs& a, int grid, int bn, cudaStream_t st);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);
cudaError_t launch_selftest_wait(int* status, cudaStream_t st);
cudaError_t gemm_prepare_single();
cudaError_t gemm_prepare_pair(int* max_clusters);
cudaError_t gemm_prepare_wide(int* max_clusters);
cudaError_t decode_prepare();

constexpr int kGemmBN = 128;   // tokens per CTA tile (single-CTA kernel)
constexpr int kGemm2BN = 256;  // tokens per CTA-pair tile
constexpr int kGemm22BN = 240; // tokens per tile of the two-strips-per-CTA pair kernel
constexpr int kDecodeBN = 16;  // tokens per decode MMA (M <= 16)
constexpr int kDecodeCtasPerSm = 4;  // decode CTAs resident per SM (four issue loops per SM)
#ifndef PATCH_DECODE_WIDE_BN
#define PATCH_DECODE_WIDE_BN 64
#endif
#ifndef PATCH_DECODE_WIDE_CTAS
#define PATCH_DECODE_WIDE_CTAS 4
#endif
constexpr int kDecodeWideBN = PATCH_DECODE_WIDE_BN;  // tokens per MMA of the decode instance for 16 < M
constexpr int kDecodeWideCtasPerSm = PATCH_DECODE_WIDE_CTAS;  // its CTAs per SM

}  // namespace patch
