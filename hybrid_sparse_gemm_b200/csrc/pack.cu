// Pack and unpack kernels: bit-packed keep/prune mask + frozen bf16 weights ->
// per-slab dense blocks or compressed 2:4 values, 2-bit position codes, and
// dense images of 2:4 slabs whose partner strip is dense.
//
// Semantics: the PATCH model cards ("llama_3.2_1b-PATCH-45Sparse", release
// paragraph and "How to use") ship only a bit-packed keep/prune mask and apply
// it by zeroing pruned weights; each tile is dense or 2:4 (method paragraph).
// The stored layout is this library's own: every record is the shared-memory
// image the tcgen05 kernels feed to the tensor core, so they load records
// with plain bulk or TMA copies.
#include "kernels.cuh"

namespace patch {

namespace {

__device__ __forceinline__ int keep_bit(uint32_t byte, int e, int bitorder) {
    return bitorder == 0 ? (byte >> (7 - e)) & 1 : (byte >> e) & 1;
}

// Zero the two metadata words (columns j, j+1) of every lane of a block.
__device__ __forceinline__ void zero_meta_words(uint8_t* meta, int j) {
    for (int lane = threadIdx.x; lane < 128; lane += blockDim.x)
        *reinterpret_cast<uint2*>(meta + lane * 16 + j * 4) = make_uint2(0u, 0u);
}

// Dense image of slab (s, b) of W (.) Mask at dst. When `count` is set the
// validation counters are updated (groups of 2:4-flagged tiles, stray zeros).
__device__ void write_dense(const PackArgs& a, int s, int b, uint8_t* dst, bool count,
                            unsigned long long& bad, unsigned long long& stray, unsigned long long& pruned) {
    const int64_t K = a.K;
    const int tiles_k = (int)(K / a.C);
    for (int q = threadIdx.x; q < 1024; q += blockDim.x) {
        const int r = q >> 3, L = (q & 7) ^ (r & 7);
        const int64_t n = (int64_t)s * kStrip + r;
        const int64_t k = (int64_t)b * kSlabK + 8 * L;
        const int64_t e0 = n * K + k;  // multiple of 8: one mask byte
        uint4 w = *reinterpret_cast<const uint4*>(a.W + e0);
        const uint32_t mb = a.bits[e0 >> 3];
        uint16_t h[8];
        memcpy(h, &w, 16);
        int kept = 0;
        for (int e = 0; e < 8; ++e) {
            const int kb = keep_bit(mb, e, a.bitorder);
            kept += kb;
            if (!kb) h[e] = 0;
        }
        if (count) {
            pruned += 8 - kept;
            if (a.flags[(n / a.R) * tiles_k + (k / a.C)]) {
                for (int g = 0; g < 2; ++g) {
                    int c = 0;
                    for (int e = 4 * g; e < 4 * g + 4; ++e) c += keep_bit(mb, e, a.bitorder);
                    bad += (c != 2);
                }
            } else {
                stray += 8 - kept;
            }
        }
        memcpy(&w, h, 16);
        *reinterpret_cast<uint4*>(dst + sw128_off(r, L)) = w;
    }
}

}  // namespace

__global__ void __launch_bounds__(256) pack_kernel(const PackArgs a) {
    __shared__ unsigned long long s_cnt[3];  // bad groups, stray zeros, pruned
    if (threadIdx.x < 3) s_cnt[threadIdx.x] = 0;
    __syncthreads();

    const int s = blockIdx.x / a.KB;
    const int b = blockIdx.x % a.KB;
    const uint32_t d = a.slab[blockIdx.x];
    uint8_t* base = a.out + slab_offset_bytes(d);
    const uint32_t mo = a.meta[s * a.KC + (b >> 1)];
    uint8_t* meta = (mo == kNoMeta) ? nullptr : a.out + (uint64_t)mo * 16;
    unsigned long long bad = 0, stray = 0, pruned = 0;

    if (!(d & kSlabSparse)) {
        write_dense(a, s, b, base, true, bad, stray, pruned);
        // A dense slab in a chunk that has a metadata block zeroes its columns.
        if (meta) zero_meta_words(meta, (b & 1) * 2);
    } else {
        const int64_t K = a.K;
        // 512 items: row r, logical 16-column quarter L (4 groups, 8 kept values).
        for (int q = threadIdx.x; q < 512; q += blockDim.x) {
            const int r = q >> 2, L = q & 3;
            const int64_t n = (int64_t)s * kStrip + r;
            const int64_t k = (int64_t)b * kSlabK + 16 * L;
            const int64_t e0 = n * K + k;
            uint16_t wv[16];
            *reinterpret_cast<uint4*>(wv) = *reinterpret_cast<const uint4*>(a.W + e0);
            *reinterpret_cast<uint4*>(wv + 8) = *reinterpret_cast<const uint4*>(a.W + e0 + 8);
            const uint32_t mb0 = a.bits[e0 >> 3], mb1 = a.bits[(e0 >> 3) + 1];
            uint16_t comp[8];
            uint32_t code = 0;
            for (int g = 0; g < 4; ++g) {
                const uint32_t mb = g < 2 ? mb0 : mb1;
                int idx[2] = {0, 0}, c = 0;
                for (int i = 0; i < 4; ++i) {
                    if (keep_bit(mb, (4 * g + i) & 7, a.bitorder)) {
                        if (c < 2) idx[c] = i;
                        ++c;
                    }
                }
                pruned += 4 - c;
                if (c != 2) {
                    ++bad;
                    idx[0] = 0;
                    idx[1] = 1;
                }
                comp[2 * g] = wv[4 * g + idx[0]];
                comp[2 * g + 1] = wv[4 * g + idx[1]];
                code |= (uint32_t)(idx[0] | (idx[1] << 2)) << (4 * g);
            }
            *reinterpret_cast<uint4*>(base + sw64_off(r, L)) = *reinterpret_cast<uint4*>(comp);
            const int kc = (b & 1) * kSlabK + 16 * L;
            *reinterpret_cast<uint16_t*>(meta + meta_lane(r, kc) * 16 + (kc >> 5) * 4 +
                                         (meta_bit(r, kc) >> 3)) = (uint16_t)code;
        }
        // The first slab of a chunk without a partner slab (K % 128 == 64)
        // zeroes the partner's columns.
        if (!(b & 1) && b + 1 >= a.KB) zero_meta_words(meta, 2);
        // A 2:4 slab whose partner strip is dense also gets a dense image for
        // the CTA-pair kernel.
        const uint32_t g = a.gemm[blockIdx.x];
        if (!(g & kSlabSparse)) {
            unsigned long long x0 = 0, x1 = 0, x2 = 0;
            write_dense(a, s, b, a.out + slab_offset_bytes(g), false, x0, x1, x2);
        }
    }

    // block reduction of the counters
    for (int o = 16; o > 0; o >>= 1) {
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
        stray += __shfl_xor_sync(0xffffffffu, stray, o);
        pruned += __shfl_xor_sync(0xffffffffu, pruned, o);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&s_cnt[0], bad);
        atomicAdd(&s_cnt[1], stray);
        atomicAdd(&s_cnt[2], pruned);
    }
    __syncthreads();
    if (threadIdx.x < 3 && s_cnt[threadIdx.x]) atomicAdd(&a.counters[threadIdx.x], s_cnt[threadIdx.x]);
}

// Decode the per-strip records back to W (.) Mask, row-major N x K.
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t* __restrict__ packed,
                                                     const uint32_t* __restrict__ slab,
                                                     const uint32_t* __restrict__ meta_tab, int KB, int KC,
                                                     int64_t K, uint16_t* __restrict__ Wm) {
    const int s = blockIdx.x / KB;
    const int b = blockIdx.x % KB;
    const uint32_t d = slab[blockIdx.x];
    const uint8_t* base = packed + slab_offset_bytes(d);
    if (!(d & kSlabSparse)) {
        for (int q = threadIdx.x; q < 1024; q += blockDim.x) {
            const int r = q >> 3, L = q & 7;
            const int64_t n = (int64_t)s * kStrip + r;
            *reinterpret_cast<uint4*>(Wm + n * K + (int64_t)b * kSlabK + 8 * L) =
                *reinterpret_cast<const uint4*>(base + sw128_off(r, L));
        }
        return;
    }
    const uint8_t* meta = packed + (uint64_t)meta_tab[s * KC + (b >> 1)] * 16;
    for (int q = threadIdx.x; q < 512; q += blockDim.x) {
        const int r = q >> 2, L = q & 3;
        const int64_t n = (int64_t)s * kStrip + r;
        uint16_t comp[8];
        *reinterpret_cast<uint4*>(comp) = *reinterpret_cast<const uint4*>(base + sw64_off(r, L));
        const int kc = (b & 1) * kSlabK + 16 * L;
        const uint32_t code = *reinterpret_cast<const uint16_t*>(
            meta + meta_lane(r, kc) * 16 + (kc >> 5) * 4 + (meta_bit(r, kc) >> 3));
        uint16_t out[16];
        for (int i = 0; i < 16; ++i) out[i] = 0;
        for (int g = 0; g < 4; ++g) {
            const uint32_t c = (code >> (4 * g)) & 15u;
            out[4 * g + (c & 3u)] = comp[2 * g];
            out[4 * g + (c >> 2)] = comp[2 * g + 1];
        }
        uint16_t* dst = Wm + n * K + (int64_t)b * kSlabK + 16 * L;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(out);
        *reinterpret_cast<uint4*>(dst + 8) = *reinterpret_cast<uint4*>(out + 8);
    }
}

}  // namespace patch
