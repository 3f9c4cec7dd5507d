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
 *   - A "strip" is 128 consecutive rows of W, a "slab" a strip times 64
 *     consecutive columns, a "chunk" two slabs (128 columns).
 *   - A slab is sparse when every mask tile it overlaps is flagged 2:4,
 *     otherwise dense.
 *   - Partners: the agreement of strips i and j is the number of slabs sparse
 *     in both. Among strips not yet paired, the two of greatest agreement
 *     become partners (ties: smallest i, then smallest j), until fewer than
 *     two remain; a strip left over is its own partner. Strips 2p and 2p+1
 *     are partners instead (the last of an odd count its own) when these
 *     pairs' agreements add up to at least those of the pairs chosen, or
 *     when there are more than 2048 strips. The pair order lists
 *     each pair's two strips (smaller first) in increasing order of its
 *     smaller strip, then the strip left over.
 *   - A slab is pair-sparse when it and its partner's slab are both sparse.
 *   - Region V, strip-major then slab: a dense slab is 16384 bytes, element
 *     (r, c) of W' (r < 128, c < 64) at byte r*128 + ((c/8) ^ (r%8))*16 +
 *     (c%8)*2; a sparse slab is 8192 bytes of the two kept bf16 of each
 *     group in ascending k, compressed element (r, j) (j < 32) at byte
 *     r*64 + ((j/8) ^ ((r/2)%4))*16 + (j%8)*2.
 *   - Region E, strip-major then chunk: one 2048-byte block per chunk that
 *     holds a sparse slab. The group starting at chunk column k of row r has
 *     the 4-bit code i0 | i1<<2 (i0 < i1 the kept positions) in the 32-bit
 *     little-endian word at byte lane*16 + (k/32)*4, lane = r%8 +
 *     8*((k%32)/16) + 16*(r/16), at bit k%16 + 16*((r/8)%2). Codes of dense
 *     or absent slabs are zero.
 *   - Region D, strip-major then slab: a 16384-byte dense image (layout of a
 *     dense slab) of every sparse slab that is not pair-sparse.
 *   - Tables (uint32): slab[s*KB+b] = (V offset/16)<<2 | first<<1 | sparse,
 *     first marking the first sparse slab of its chunk;
 *     meta[s*KC+c] = E offset/16 or 0xFFFFFFFF (KC = ceil(KB/2));
 *     gemm[s*KB+b] = (offset/16)<<2 | load_meta<<1 | pair_sparse, where the
 *     offset is the V record when the slab is pair-sparse or dense and the
 *     D image otherwise, and load_meta marks the first pair-sparse slab of
 *     its chunk.
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

static int64_t or_agreement(const uint8_t* flags, int64_t K, int R, int C, int64_t i, int64_t j) {
    int64_t agree = 0;
    for (int64_t b = 0; b < K / OR_SLAB; ++b)
        agree += or_slab_sparse(flags, K, R, C, i, b) && or_slab_sparse(flags, K, R, C, j, b);
    return agree;
}

/* partner[s] of every strip, by the rule above; returns 0. */
static int or_partners(const uint8_t* flags, int64_t N, int64_t K, int R, int C, int64_t* partner) {
    int64_t S = N / OR_STRIP, chosen = 0, fixed = 0;
    for (int64_t s = 0; s + 1 < S; s += 2) fixed += or_agreement(flags, K, R, C, s, s + 1);
    for (int64_t s = 0; s < S; ++s) partner[s] = -1;
    for (;;) {
        int64_t bi = -1, bj = -1, best = -1;
        for (int64_t i = 0; i < S; ++i) {
            if (partner[i] >= 0) continue;
            for (int64_t j = i + 1; j < S && S <= 2048; ++j) {
                if (partner[j] >= 0) continue;
                int64_t agree = or_agreement(flags, K, R, C, i, j);
                if (agree > best) { /* strictly greater: the first (i, j) wins a tie */
                    best = agree;
                    bi = i;
                    bj = j;
                }
            }
        }
        if (bi < 0) break;
        partner[bi] = bj;
        partner[bj] = bi;
        chosen += best;
    }
    if (S > 2048 || fixed >= chosen)
        for (int64_t s = 0; s < S; ++s) partner[s] = -1;
    for (int64_t s = 0; s + 1 < S; s += 2)
        if (partner[s] < 0 && partner[s + 1] < 0) {
            partner[s] = s + 1;
            partner[s + 1] = s;
        }
    for (int64_t s = 0; s < S; ++s)
        if (partner[s] < 0) partner[s] = s;
    return 0;
}

/* The pair order: pair i is order[2i], order[2i+1]. Returns 0 or -1. */
int oracle_pair_order(int64_t N, int64_t K, const uint8_t* flags, int R, int C, int32_t* order) {
    int64_t S = N / OR_STRIP, n = 0;
    int64_t* partner = (int64_t*)malloc(sizeof(int64_t) * (size_t)(S > 0 ? S : 1));
    if (!partner || or_partners(flags, N, K, R, C, partner) != 0) {
        free(partner);
        return -1;
    }
    for (int64_t s = 0; s < S; ++s)
        if (partner[s] > s) {
            order[n++] = (int32_t)s;
            order[n++] = (int32_t)partner[s];
        }
    for (int64_t s = 0; s < S; ++s)
        if (partner[s] == s) order[n++] = (int32_t)s;
    free(partner);
    return 0;
}

static int or_pair_sparse(const uint8_t* flags, int64_t K, int R, int C, const int64_t* partner,
                          int64_t s, int64_t b) {
    return or_slab_sparse(flags, K, R, C, s, b) && or_slab_sparse(flags, K, R, C, partner[s], b);
}

/* Fills the three tables and returns the total packed byte count (-1 when
 * out of memory). */
int64_t oracle_pack_table(int64_t N, int64_t K, const uint8_t* flags, int R, int C,
                          uint32_t* slab, uint32_t* meta, uint32_t* gemm) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB, KC = (KB + 1) / 2, off = 0;
    int64_t* partner = (int64_t*)malloc(sizeof(int64_t) * (size_t)(S > 0 ? S : 1));
    if (!partner || or_partners(flags, N, K, R, C, partner) != 0) {
        free(partner);
        return -1;
    }
    /* region V */
    for (int64_t s = 0; s < S; ++s)
        for (int64_t b = 0; b < KB; ++b) {
            int sp = or_slab_sparse(flags, K, R, C, s, b);
            int first = sp && (b % 2 == 0 || !or_slab_sparse(flags, K, R, C, s, b - 1));
            slab[s * KB + b] = (uint32_t)((off / 16) << 2) | (uint32_t)(first << 1) | (uint32_t)sp;
            off += sp ? 8192 : 16384;
        }
    /* region E */
    for (int64_t s = 0; s < S; ++s)
        for (int64_t c = 0; c < KC; ++c) {
            int any = 0;
            for (int64_t b = 2 * c; b < 2 * c + 2 && b < KB; ++b)
                any |= or_slab_sparse(flags, K, R, C, s, b);
            if (any) {
                meta[s * KC + c] = (uint32_t)(off / 16);
                off += 2048;
            } else {
                meta[s * KC + c] = 0xFFFFFFFFu;
            }
        }
    /* region D and the tensor-core table */
    for (int64_t s = 0; s < S; ++s)
        for (int64_t b = 0; b < KB; ++b) {
            int sp = or_slab_sparse(flags, K, R, C, s, b);
            int psp = or_pair_sparse(flags, K, R, C, partner, s, b);
            int64_t a_off;
            if (sp && !psp) {
                a_off = off;
                off += 16384;
            } else {
                a_off = (int64_t)(slab[s * KB + b] >> 2) * 16;
            }
            int load_meta = psp && (b % 2 == 0 || !or_pair_sparse(flags, K, R, C, partner, s, b - 1));
            gemm[s * KB + b] = (uint32_t)((a_off / 16) << 2) | (uint32_t)(load_meta << 1) |
                               (uint32_t)psp;
        }
    free(partner);
    return off;
}

static void or_put16(uint8_t* p, uint16_t v) {
    p[0] = (uint8_t)(v & 0xff);
    p[1] = (uint8_t)(v >> 8);
}

static void or_dense_image(const uint16_t* W, const uint8_t* keep, int64_t K, int64_t s, int64_t b,
                           uint8_t* base) {
    int64_t k0 = b * OR_SLAB;
    for (int r = 0; r < OR_STRIP; ++r) {
        int64_t n = s * OR_STRIP + r;
        for (int c = 0; c < OR_SLAB; ++c) {
            uint16_t v = keep[n * K + k0 + c] ? W[n * K + k0 + c] : 0;
            or_put16(base + (int64_t)r * 128 + (((c / 8) ^ (r % 8)) * 16) + (c % 8) * 2, v);
        }
    }
}

/* Writes the packed bytes. The mask must already be valid (every group of a
 * 2:4-flagged tile keeps exactly two); returns -1 otherwise. */
int oracle_pack(const uint16_t* W, const uint8_t* keep, int64_t N, int64_t K,
                const uint32_t* slab, const uint32_t* meta, const uint32_t* gemm, uint8_t* out) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB, KC = (KB + 1) / 2;
    for (int64_t s = 0; s < S; ++s)
        for (int64_t c = 0; c < KC; ++c)
            if (meta[s * KC + c] != 0xFFFFFFFFu) memset(out + (int64_t)meta[s * KC + c] * 16, 0, 2048);
    for (int64_t s = 0; s < S; ++s) {
        for (int64_t b = 0; b < KB; ++b) {
            uint8_t* base = out + (int64_t)(slab[s * KB + b] >> 2) * 16;
            int64_t k0 = b * OR_SLAB;
            if (!(slab[s * KB + b] & 1)) {
                or_dense_image(W, keep, K, s, b, base);
                continue;
            }
            if (!(gemm[s * KB + b] & 1))
                or_dense_image(W, keep, K, s, b, out + (int64_t)(gemm[s * KB + b] >> 2) * 16);
            uint32_t mo = meta[s * KC + b / 2];
            if (mo == 0xFFFFFFFFu) return -1;
            uint8_t* mb = out + (int64_t)mo * 16;
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
                        or_put16(base + (int64_t)r * 64 + (((j / 8) ^ ((r / 2) % 4)) * 16) + (j % 8) * 2,
                                 W[n * K + k0 + 4 * g + idx[t]]);
                    }
                    int code = idx[0] | (idx[1] << 2);
                    int kc = (int)((b % 2) * OR_SLAB + 4 * g); /* column inside the chunk */
                    int lane = (r % 8) + 8 * ((kc % 32) / 16) + 16 * (r / 16);
                    int bit = (kc % 16) + 16 * ((r / 8) % 2);
                    uint8_t* wp = mb + lane * 16 + (kc / 32) * 4;
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

/* Decodes region V (with the metadata of region E) back to W' (N x K bf16
 * bits). */
int oracle_unpack(const uint8_t* packed, const uint32_t* slab, const uint32_t* meta, int64_t N,
                  int64_t K, uint16_t* Wm) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB, KC = (KB + 1) / 2;
    for (int64_t s = 0; s < S; ++s) {
        for (int64_t b = 0; b < KB; ++b) {
            const uint8_t* base = packed + (int64_t)(slab[s * KB + b] >> 2) * 16;
            int64_t k0 = b * OR_SLAB;
            if (!(slab[s * KB + b] & 1)) {
                for (int r = 0; r < OR_STRIP; ++r)
                    for (int c = 0; c < OR_SLAB; ++c) {
                        int64_t at = (int64_t)r * 128 + (((c / 8) ^ (r % 8)) * 16) + (c % 8) * 2;
                        Wm[(s * OR_STRIP + r) * K + k0 + c] =
                            (uint16_t)(base[at] | (base[at + 1] << 8));
                    }
                continue;
            }
            uint32_t mo = meta[s * KC + b / 2];
            if (mo == 0xFFFFFFFFu) return -1;
            const uint8_t* mb = packed + (int64_t)mo * 16;
            for (int r = 0; r < OR_STRIP; ++r) {
                int64_t n = s * OR_STRIP + r;
                for (int g = 0; g < OR_SLAB / 4; ++g) {
                    int kc = (int)((b % 2) * OR_SLAB + 4 * g);
                    int lane = (r % 8) + 8 * ((kc % 32) / 16) + 16 * (r / 16);
                    const uint8_t* wp = mb + lane * 16 + (kc / 32) * 4;
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

/* Decodes the tensor-core view: for every slab, the record the gemm table
 * points at, back to W' (checks that dense images equal W' too). */
int oracle_unpack_gemm(const uint8_t* packed, const uint32_t* gemm, const uint32_t* meta,
                       int64_t N, int64_t K, uint16_t* Wm) {
    int64_t S = N / OR_STRIP, KB = K / OR_SLAB, KC = (KB + 1) / 2;
    uint32_t* one = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)KB);
    if (!one) return -1;
    for (int64_t s = 0; s < S; ++s) {
        for (int64_t b = 0; b < KB; ++b) one[b] = gemm[s * KB + b];
        /* decode strip s as a one-strip matrix through oracle_unpack */
        uint16_t* dst = Wm + s * OR_STRIP * K;
        int rc = oracle_unpack(packed, one, meta + s * KC, OR_STRIP, K, dst);
        if (rc != 0) {
            free(one);
            return rc;
        }
    }
    free(one);
    return 0;
}
