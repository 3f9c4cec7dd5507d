/*
 * CPU oracle for the PATCH hybrid dense / 2:4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link,
 * load or call this file: only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark do. It shares no code, header, table or constant with
 * the CUDA library; the two sides meet only through seeded inputs.
 *
 * What it computes, and where the pages fix it:
 *
 *  - The mask is a binary keep/prune mask over the frozen weights, shipped
 *    bit-packed (model card "llama_3.2_1b-PATCH-45Sparse", method paragraph
 *    and "How to use"; same text on "gemma_3_1b-MaskLLM-50Sparse").
 *  - Applying it zeroes the pruned weights in place ("How to use",
 *    apply_patch_mask): the effective weight is W' = W (.) Mask.
 *  - Each weight tile is either dense (0% sparsity) or 2:4 sparse (two kept
 *    in every group of four) (method paragraph; abstract of "PATCH:
 *    Learnable Tile-level Hybrid Sparsity for LLMs").
 *  - Mask tile 128x128; hardware tiles 128x128 / 128x64 / 64x128 / 64x64
 *    (llama card, "Training hyper-parameters" table, mask tile size row).
 *  - Global sparsity is continuous in [0%, 50%] (abstract); with exactly two
 *    of four kept in a 2:4 tile and none pruned in a dense tile it equals
 *    one half of the area fraction of 2:4 tiles.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - 2:4 groups run along K (the reduction axis, columns of W[N,K]).
 *  - The mask is row-major over W[N,K]; bit b sits in byte b>>3 at bit
 *    7-(b&7) (MSB first, numpy packbits default) or at bit b&7 (LSB first).
 *  - Y = X W'^T with fp32 products and an fp32 running sum over ascending k,
 *    rounded once to bf16 (round to nearest, ties to even).
 *
 * The packed format is this library's own (the pages give none). Its
 * independent restatement here lets tests check the GPU pack byte by byte:
 *   - A "strip" is 128 consecutive rows of W; a "slab" is a strip times 64
 *     consecutive columns. Slabs are stored strip-major, K ascending.
 *   - A slab is sparse when every mask tile it overlaps is flagged 2:4,
 *     otherwise dense.
 *   - Dense slab: 16384 bytes, element (r, c) of W' (r < 128, c < 64) at
 *     byte r*128 + ((c/8) ^ (r%8))*16 + (c%8)*2.
 *   - Sparse slab values: 8192 bytes, the two kept bf16 of each group in
 *     ascending k; compressed element (r, j) (j < 32) at byte
 *     r*64 + ((j/8) ^ ((r/2)%4))*16 + (j%8)*2.
 *   - Metadata: one 2048-byte block per (strip, 128-column chunk) that holds
 *     at least one sparse slab, stored right after the values of the first
 *     sparse slab in the chunk. The group that starts at chunk column k of
 *     row r has the 4-bit code i0 | i1<<2 (i0 < i1 the kept positions) in
 *     32-bit little-endian word (lane, k/32) at byte lane*16 + (k/32)*4, with
 *     lane = r%8 + 8*((k%32)/16) + 16*(r/16), at bit k%16 + 16*((r/8)%2).
 *     Codes of dense slabs in the chunk are zero.
 *   - Slab table: one uint32 per slab, (byte_offset/16)<<2 | has_meta<<1 |
 *     sparse.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_STRIP 128
#define OR_SLAB 64
#define OR_CHUNK 128

/* ---- bf16 <-> fp32 ------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32, so widening is exact. */
static float or_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round to nearest, ties to even; NaN stays NaN (quiet bit set). */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

void oracle_round_bf16(const float* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(y[i]);
}

/* ---- mask ---------------------------------------------------------------- */

/* keep bit for flat element index idx of the row-major N x K mask. */
static int or_bit(const uint8_t* bits, int64_t idx, int bitorder) {
    int pos = bitorder == 0 ? 7 - (int)(idx & 7) : (int)(idx & 7);
    return (bits[idx >> 3] >> pos) & 1;
}

void oracle_expand_mask(const uint8_t* bits, int64_t N, int64_t K, int bitorder,
                        uint8_t* keep) {
    for (int64_t i = 0; i < N * K; ++i) keep[i] = (uint8_t)or_bit(bits, i, bitorder);
}

/* Number of 2:4 groups (inside tiles flagged 2:4) whose kept count is not
 * exactly two; *stray_zeros gets the pruned elements found in dense tiles. */
int64_t oracle_check_tiles(const uint8_t* keep, int64_t N, int64_t K,
                           const uint8_t* flags, int R, int C, int64_t* stray_zeros) {
    int64_t bad = 0, stray = 0, tiles_k = K / C;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; k += 4) {
            int sparse = flags[(n / R) * tiles_k + (k / C)];
            int kept = keep[n * K + k] + keep[n * K + k + 1] + keep[n * K + k + 2] +
                       keep[n * K + k + 3];
            if (sparse) {
                if (kept != 2) ++bad;
            } else {
                stray += 4 - kept;
            }
        }
    }
    if (stray_zeros) *stray_zeros = stray;
    return bad;
}

/* Measured mask sparsity: pruned elements over all elements. */
double oracle_sparsity(const uint8_t* keep, int64_t N, int64_t K) {
    int64_t zeros = 0;
    for (int64_t i = 0; i < N * K; ++i) zeros += keep[i] == 0;
    return (double)zeros / (double)(N * K);
}

/* W' = W (.) Mask, pruned entries become +0.0 (bf16 bit pattern 0). */
void oracle_apply_mask(const uint16_t* W, const uint8_t* keep, int64_t N, int64_t K,
                       uint16_t* Wm) {
    for (int64_t i = 0; i < N * K; ++i) Wm[i] = keep[i] ? W[i] : (uint16_t)0;
}

/* ---- the linear layer ---------------------------------------------------- */

/* Y[i][n] = sum_{k ascending} fp32(X[rows[i]][k]) * fp32(W'[n][k]), fp32 sum.
 * rows == NULL means rows 0..nrows-1. Y is nrows x N, fp32. Rows of the
 * product are independent, so any subset is exact. */
void oracle_linear_f32(const uint16_t* X, int64_t M, int64_t K, const uint16_t* Wm,
                       int64_t N, const int64_t* rows, int64_t nrows, float* Y) {
    (void)M;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows ? rows[i] : i;
            const uint16_t* x = X + m * K;
            const uint16_t* w = Wm + n * K;
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float prod = or_bf16_to_f32(x[k]) * or_bf16_to_f32(w[k]);
                acc = acc + prod;
            }
            Y[i * N + n] = acc;
        }
    }
}

/* sum_k |x_k * w_k| per output, the scale of the error bounds. */
void oracle_abs_scale(const uint16_t* X, int64_t K, const uint16_t* Wm, int64_t N,
                      const int64_t* rows, int64_t nrows, double* S) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows ? rows[i] : i;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += fabs((double)or_bf16_to_f32(X[m * K + k]) *
                          (double)or_bf16_to_f32(Wm[n * K + k]));
            S[i * N + n] = s;
        }
    }
}

/* ---- packed format (independent restatement) ----------------------------- */

static int or_slab_sparse(const uint8_t* flags, int64_t K, int R, int C, int64_t s,
                          int64_t b) {
    int64_t tiles_k = K / C;
    int64_t col = (b * OR_SLAB) / C;
    for (int64_t r0 = s * OR_STRIP; r0 < (s + 1) * OR_STRIP; r0 += R)
        if (!flags[(r0 / R) * tiles_k + col]) return 0;
    return 1;
}

/* Fills table[S*KB] and returns the total packed byte count. */
int64_t oracle_pack_table(int64_t N, int64_t K, const uint8_t* flags, int R, int C,
                          uint32_t* table) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB, off = 0;
    for (int64_t s = 0; s < S; ++s) {
        int meta_done_chunk = -1;
        for (int64_t b = 0; b < KB; ++b) {
            int sp = or_slab_sparse(flags, K, R, C, s, b);
            int has_meta = 0;
            int64_t chunk = b / 2;
            if (sp && meta_done_chunk != (int)chunk) {
                has_meta = 1;
                meta_done_chunk = (int)chunk;
            }
            table[s * KB + b] = (uint32_t)((off / 16) << 2) | (uint32_t)(has_meta << 1) |
                                (uint32_t)sp;
            off += sp ? 8192 + (has_meta ? 2048 : 0) : 16384;
        }
    }
    return off;
}

/* Writes the packed bytes. The mask must already be valid (every group of a
 * 2:4-flagged tile keeps exactly two); returns -1 otherwise. */
int oracle_pack(const uint16_t* W, const uint8_t* keep, int64_t N, int64_t K,
                const uint8_t* flags, int R, int C, const uint32_t* table, uint8_t* out) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB;
    for (int64_t s = 0; s < S; ++s) {
        uint8_t* meta = NULL;
        int64_t meta_chunk = -1;
        for (int64_t b = 0; b < KB; ++b) {
            uint32_t d = table[s * KB + b];
            uint8_t* base = out + (int64_t)(d >> 2) * 16;
            int sp = d & 1;
            int64_t k0 = b * OR_SLAB;
            if (!sp) {
                for (int r = 0; r < OR_STRIP; ++r) {
                    int64_t n = s * OR_STRIP + r;
                    for (int c = 0; c < OR_SLAB; ++c) {
                        uint16_t v = keep[n * K + k0 + c] ? W[n * K + k0 + c] : 0;
                        int64_t at = (int64_t)r * 128 + (((c / 8) ^ (r % 8)) * 16) + (c % 8) * 2;
                        base[at] = (uint8_t)(v & 0xff);
                        base[at + 1] = (uint8_t)(v >> 8);
                    }
                }
                continue;
            }
            if (d & 2) {
                meta = base + 8192;
                meta_chunk = b / 2;
                memset(meta, 0, 2048);
            }
            if (meta == NULL || meta_chunk != b / 2) return -1;
            for (int r = 0; r < OR_STRIP; ++r) {
                int64_t n = s * OR_STRIP + r;
                for (int g = 0; g < OR_SLAB / 4; ++g) {
                    int idx[2], cnt = 0;
                    for (int i = 0; i < 4; ++i)
                        if (keep[n * K + k0 + 4 * g + i]) {
                            if (cnt < 2) idx[cnt] = i;
                            ++cnt;
                        }
                    if (cnt != 2) return -1;
                    for (int t = 0; t < 2; ++t) {
                        int j = 2 * g + t;
                        uint16_t v = W[n * K + k0 + 4 * g + idx[t]];
                        int64_t at = (int64_t)r * 64 + (((j / 8) ^ ((r / 2) % 4)) * 16) + (j % 8) * 2;
                        base[at] = (uint8_t)(v & 0xff);
                        base[at + 1] = (uint8_t)(v >> 8);
                    }
                    int code = idx[0] | (idx[1] << 2);
                    int kc = (int)((b % 2) * OR_SLAB + 4 * g); /* column inside the chunk */
                    int lane = (r % 8) + 8 * ((kc % 32) / 16) + 16 * (r / 16);
                    int word = kc / 32;
                    int bit = (kc % 16) + 16 * ((r / 8) % 2);
                    uint8_t* wp = meta + lane * 16 + word * 4;
                    uint32_t wv = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                                  ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
                    wv |= (uint32_t)code << bit;
                    wp[0] = (uint8_t)wv;
                    wp[1] = (uint8_t)(wv >> 8);
                    wp[2] = (uint8_t)(wv >> 16);
                    wp[3] = (uint8_t)(wv >> 24);
                }
            }
        }
    }
    return 0;
}

/* Decodes packed bytes back to W' (N x K bf16 bits). */
int oracle_unpack(const uint8_t* packed, const uint32_t* table, int64_t N, int64_t K,
                  uint16_t* Wm) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB;
    for (int64_t s = 0; s < S; ++s) {
        const uint8_t* meta = NULL;
        int64_t meta_chunk = -1;
        for (int64_t b = 0; b < KB; ++b) {
            uint32_t d = table[s * KB + b];
            const uint8_t* base = packed + (int64_t)(d >> 2) * 16;
            int64_t k0 = b * OR_SLAB;
            if (!(d & 1)) {
                for (int r = 0; r < OR_STRIP; ++r)
                    for (int c = 0; c < OR_SLAB; ++c) {
                        int64_t at = (int64_t)r * 128 + (((c / 8) ^ (r % 8)) * 16) + (c % 8) * 2;
                        Wm[(s * OR_STRIP + r) * K + k0 + c] =
                            (uint16_t)(base[at] | (base[at + 1] << 8));
                    }
                continue;
            }
            if (d & 2) {
                meta = base + 8192;
                meta_chunk = b / 2;
            }
            if (meta == NULL || meta_chunk != b / 2) return -1;
            for (int r = 0; r < OR_STRIP; ++r) {
                int64_t n = s * OR_STRIP + r;
                for (int g = 0; g < OR_SLAB / 4; ++g) {
                    int kc = (int)((b % 2) * OR_SLAB + 4 * g);
                    int lane = (r % 8) + 8 * ((kc % 32) / 16) + 16 * (r / 16);
                    const uint8_t* wp = meta + lane * 16 + (kc / 32) * 4;
                    uint32_t wv = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                                  ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
                    int code = (int)((wv >> ((kc % 16) + 16 * ((r / 8) % 2))) & 0xf);
                    int i0 = code & 3, i1 = code >> 2;
                    if (i0 >= i1) return -1;
                    for (int i = 0; i < 4; ++i) Wm[n * K + k0 + 4 * g + i] = 0;
                    for (int t = 0; t < 2; ++t) {
                        int j = 2 * g + t;
                        int64_t at = (int64_t)r * 64 + (((j / 8) ^ ((r / 2) % 4)) * 16) + (j % 8) * 2;
                        Wm[n * K + k0 + 4 * g + (t ? i1 : i0)] =
                            (uint16_t)(base[at] | (base[at + 1] << 8));
                    }
                }
            }
        }
    }
    return 0;
}
