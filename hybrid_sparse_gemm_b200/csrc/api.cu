// Host runtime behind the C ABI in patch_hybrid.h: argument checks, the slab
// tables, the cost-balanced persistent schedules, tensor maps and launches.
//
// Every tensor-core launch runs a group of packed linears that share M; a
// single patch_linear call runs the handle's own one-member group.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <queue>
#include <string>
#include <thread>
#include <vector>

#include "kernels.cuh"
#include "patch_hybrid.h"

using namespace patch;

// Smallest K-part (packed bytes) of the decode kernel's 64-token instance in
// a group (a macro so that other sizes can be measured).
#ifndef PATCH_DECODE_WIDE_PART_KB
#define PATCH_DECODE_WIDE_PART_KB 512.0
#endif

namespace {

thread_local std::string g_err;

patch_status fail(patch_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

patch_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PATCH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define PATCH_CUDA(call)                                    \
    do {                                                    \
        cudaError_t e_ = (call);                            \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

patch_status check_shape(int64_t N, int64_t K, int tile_rows, int tile_cols) {
    const bool shape_ok = (tile_rows == 128 || tile_rows == 64) && (tile_cols == 128 || tile_cols == 64);
    if (!shape_ok)
        return fail(PATCH_ERR_SHAPE, "tile shape %dx%d is not one of 128x128, 128x64, 64x128, 64x64", tile_rows,
                    tile_cols);
    if (N <= 0 || K <= 0) return fail(PATCH_ERR_SHAPE, "N and K must be positive");
    if (N % kStrip || K % kSlabK || N % tile_rows || K % tile_cols)
        return fail(PATCH_ERR_SHAPE,
                    "need N %% 128 == 0, K %% 64 == 0 and both divisible by the tile (N=%lld K=%lld)",
                    (long long)N, (long long)K);
    if (N > (1 << 24) || K > (1 << 24) || N * K > ((int64_t)1 << 36))
        return fail(PATCH_ERR_SHAPE, "weight too large");
    return PATCH_OK;
}

patch_status check_flags(const uint8_t* flags, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        if (flags[i] > 1)
            return fail(PATCH_ERR_ARG, "tile flag %lld is %d, must be 0 or 1", (long long)i, (int)flags[i]);
    return PATCH_OK;
}

struct DeviceInfo {
    int sms = 0;
    int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair kernel
    int wide_clusters = 0;  // co-resident CTA pairs of the two-strips-per-CTA kernel
};
std::mutex g_dev_mu;
std::map<int, DeviceInfo> g_dev;

patch_status prepare_device(int* dev_out, DeviceInfo* info_out) {
    int dev = 0;
    PATCH_CUDA(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        int major = 0, sms = 0;
        PATCH_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        PATCH_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
        if (major != 10)
            return fail(PATCH_ERR_UNSUPPORTED, "device %d has compute capability %d.x, need 10.x", dev, major);
        DeviceInfo di;
        di.sms = sms;
        PATCH_CUDA(gemm_prepare_single());
        PATCH_CUDA(gemm_prepare_pair(&di.pair_clusters));
        PATCH_CUDA(gemm_prepare_wide(&di.wide_clusters));
        if (di.wide_clusters <= 0) di.wide_clusters = 1;
        PATCH_CUDA(decode_prepare());
        if (di.pair_clusters <= 0) di.pair_clusters = 1;
        it = g_dev.emplace(dev, di).first;
    }
    *dev_out = dev;
    *info_out = it->second;
    return PATCH_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

patch_status get_encode() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return fail(PATCH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    return PATCH_OK;
}

// 2-D bf16 tensor map: `rows` rows of `cols` elements (row pitch cols*2 bytes),
// box of box_cols x box_rows.
patch_status encode_2d(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int box_cols, int box_rows,
                       CUtensorMapSwizzle swizzle) {
    patch_status st = get_encode();
    if (st != PATCH_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PATCH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PATCH_OK;
}

struct WorkList {
    int grid = 0;         // CTAs (single, decode) or CTA pairs (pair kernel)
    int* off = nullptr;   // device, grid + 1
    int* work = nullptr;  // device, units
    int* host = nullptr;  // pinned host copy the upload reads from (kept until the group is freed)
    cudaEvent_t ready = nullptr;      // recorded after the upload on the stream that built it
    cudaStream_t made_on = nullptr;
    std::atomic<bool> done{false};    // the upload is known to have completed
};

// Split-K workspace of the decode kernel for one group and one stream: per
// member, partial sums [S][P][128][16] fp32 (NULL when P == 1) and per-strip
// arrival counters that the kernel re-arms to zero.
struct DecodeWs {
    float* partial[kMaxGroup] = {};       // 16-token partials (M <= 16)
    float* partial_wide[kMaxGroup] = {};  // kDecodeWideBN-token partials, allocated on the first call with M > 16
    unsigned* counters[kMaxGroup] = {};
    int S[kMaxGroup] = {};
};

// Host copy of the three tables and the derived per-strip costs.
struct Plan {
    int S = 0, KB = 0, KC = 0;
    std::vector<uint32_t> slab, meta, gemm;
    std::vector<int> order;                     // strips by pair position: pair i = (order[2i], order[2i+1])
    std::vector<uint32_t> pgemm, pmeta;         // gemm and meta with rows in pair-position order
    std::vector<double> strip_cost, pair_cost;  // tensor-core time: dense slab 1, 2:4 slab 1/2 (pair_cost by pair)
    std::vector<double> adj_pair_cost;          // the same for strips (2q, 2q+1): the row-partition estimate
    std::vector<double> strip_bytes;            // bytes the decode kernel streams per strip
    int64_t bytes = 0, sparse = 0, pair_sparse = 0, meta_blocks = 0, images = 0;
};

// Partners of the CTA-pair kernels. One pair MMA covers two strips and must
// be dense or 2:4 for both, so a 2:4 slab whose partner's slab is dense runs
// from a dense image at dense cost. Strips are therefore paired by agreement:
// score(i, j) = slabs that are 2:4 in both; repeatedly pair the two unpaired
// strips of highest score (ties: smallest i, then smallest j); pairs go in
// the order of their first strip, an odd strip out last (its own partner).
// If the fixed pairs (2p, 2p+1) score at least as much in total, they are
// kept (order 0, 1, 2, ...: so strips of equal patterns, all dense or all
// 2:4, keep it), and so does a linear of more than kMaxPairedStrips strips
// (the scores would take S^2 / 2 entries).
constexpr int kMaxPairedStrips = 2048;

std::vector<int> pair_order(const std::vector<uint8_t>& sp, int S, int KB) {
    if (S > kMaxPairedStrips) {
        std::vector<int> order(S);
        for (int s = 0; s < S; ++s) order[s] = s;
        return order;
    }
    const int words = (KB + 63) / 64;
    std::vector<uint64_t> bits((size_t)S * words, 0);
    for (int s = 0; s < S; ++s)
        for (int b = 0; b < KB; ++b)
            if (sp[(size_t)s * KB + b]) bits[(size_t)s * words + b / 64] |= 1ull << (b % 64);
    struct Cand {
        int score, i, j;
    };
    std::vector<Cand> cand;
    cand.reserve((size_t)S * (S - 1) / 2);
    for (int i = 0; i < S; ++i)
        for (int j = i + 1; j < S; ++j) {
            int sc = 0;
            for (int w = 0; w < words; ++w)
                sc += __builtin_popcountll(bits[(size_t)i * words + w] & bits[(size_t)j * words + w]);
            cand.push_back({sc, i, j});
        }
    std::sort(cand.begin(), cand.end(), [](const Cand& x, const Cand& y) {
        return x.score != y.score ? x.score > y.score : x.i != y.i ? x.i < y.i : x.j < y.j;
    });
    std::vector<uint8_t> used(S, 0);
    std::vector<std::pair<int, int>> pairs;
    int64_t greedy = 0, fixed = 0;
    for (const Cand& c : cand) {
        if (used[c.i] || used[c.j]) continue;
        used[c.i] = used[c.j] = 1;
        pairs.push_back({c.i, c.j});
        greedy += c.score;
    }
    for (int i = 0; i + 1 < S; i += 2)
        for (int w = 0; w < words; ++w)
            fixed += __builtin_popcountll(bits[(size_t)i * words + w] & bits[(size_t)(i + 1) * words + w]);
    if (fixed >= greedy) {
        std::vector<int> order(S);
        for (int s = 0; s < S; ++s) order[s] = s;
        return order;
    }
    std::sort(pairs.begin(), pairs.end());
    std::vector<int> order;
    order.reserve(S);
    for (const auto& pr : pairs) {
        order.push_back(pr.first);
        order.push_back(pr.second);
    }
    for (int s = 0; s < S; ++s)
        if (!used[s]) order.push_back(s);
    return order;
}

// Region V (every slab), region E (a metadata block per chunk holding a 2:4
// slab), region D (dense images of 2:4 slabs whose partner strip is dense).
void build_plan(Plan& p, int64_t N, int64_t K, int R, int C, const uint8_t* flags) {
    p.S = (int)(N / kStrip);
    p.KB = (int)(K / kSlabK);
    p.KC = (p.KB + 1) / 2;
    const int64_t tiles_k = K / C;
    std::vector<uint8_t> sp((size_t)p.S * p.KB);
    for (int s = 0; s < p.S; ++s)
        for (int b = 0; b < p.KB; ++b) {
            bool all = true;
            for (int r0 = s * kStrip; r0 < (s + 1) * kStrip; r0 += R)
                all = all && flags[(int64_t)(r0 / R) * tiles_k + ((int64_t)b * kSlabK) / C] != 0;
            sp[(size_t)s * p.KB + b] = all;
        }
    auto is_sp = [&](int s, int b) { return sp[(size_t)s * p.KB + b] != 0; };
    p.order = pair_order(sp, p.S, p.KB);
    std::vector<int> partner_of(p.S);
    for (int q = 0; q < p.S; ++q) partner_of[p.order[q]] = (q ^ 1) < p.S ? p.order[q ^ 1] : p.order[q];
    auto pair_sp = [&](int s, int b) { return is_sp(s, b) && is_sp(partner_of[s], b); };
    p.slab.assign((size_t)p.S * p.KB, 0u);
    p.meta.assign((size_t)p.S * p.KC, kNoMeta);
    p.gemm.assign((size_t)p.S * p.KB, 0u);
    p.strip_cost.assign(p.S, 0.0);
    p.pair_cost.assign((p.S + 1) / 2, 0.0);
    p.adj_pair_cost.assign((p.S + 1) / 2, 0.0);
    p.strip_bytes.assign(p.S, 0.0);
    int64_t off = 0;
    for (int s = 0; s < p.S; ++s)
        for (int b = 0; b < p.KB; ++b) {
            const bool x = is_sp(s, b);
            const bool first = x && (b % 2 == 0 || !is_sp(s, b - 1));
            p.slab[(size_t)s * p.KB + b] =
                (uint32_t)((off / 16) << 2) | (first ? kSlabFirst : 0u) | (x ? kSlabSparse : 0u);
            off += x ? kSparseValBytes : kDenseSlabBytes;
            p.sparse += x;
            p.strip_cost[s] += x ? 0.5 : 1.0;
            p.strip_bytes[s] += x ? kSparseValBytes : kDenseSlabBytes;
        }
    for (int s = 0; s < p.S; ++s)
        for (int c = 0; c < p.KC; ++c) {
            bool any = is_sp(s, 2 * c) || (2 * c + 1 < p.KB && is_sp(s, 2 * c + 1));
            if (any) {
                p.meta[(size_t)s * p.KC + c] = (uint32_t)(off / 16);
                off += kMetaBytes;
                ++p.meta_blocks;
                p.strip_bytes[s] += kMetaBytes;
            }
        }
    for (int s = 0; s < p.S; ++s)
        for (int b = 0; b < p.KB; ++b) {
            const bool x = is_sp(s, b), px = pair_sp(s, b);
            int64_t a_off;
            if (x && !px) {
                a_off = off;
                off += kDenseSlabBytes;
                ++p.images;
            } else {
                a_off = (int64_t)slab_offset_bytes(p.slab[(size_t)s * p.KB + b]);
            }
            const bool first = px && (b % 2 == 0 || !pair_sp(s, b - 1));
            p.gemm[(size_t)s * p.KB + b] =
                (uint32_t)((a_off / 16) << 2) | (first ? kSlabFirst : 0u) | (px ? kSlabSparse : 0u);
            p.pair_sparse += px;
            if ((s & 1) == 0) {
                const int t = (s + 1) < p.S ? s + 1 : s;
                p.adj_pair_cost[s / 2] += (x && is_sp(t, b)) ? 0.5 : 1.0;
            }
        }
    for (int i = 0; i < (p.S + 1) / 2; ++i)
        for (int b = 0; b < p.KB; ++b) p.pair_cost[i] += pair_sp(p.order[2 * i], b) ? 0.5 : 1.0;
    p.pgemm.resize(p.gemm.size());
    p.pmeta.resize(p.meta.size());
    for (int q = 0; q < p.S; ++q) {
        std::copy_n(p.gemm.begin() + (size_t)p.order[q] * p.KB, p.KB, p.pgemm.begin() + (size_t)q * p.KB);
        std::copy_n(p.meta.begin() + (size_t)p.order[q] * p.KC, p.KC, p.pmeta.begin() + (size_t)q * p.KC);
    }
    p.bytes = off;
}

// Decode K-parts per strip: the fewest parts that keep the per-CTA load within
// a few percent of the best split, each part costing one extra epilogue.
int choose_decode_parts(int S, int KC, int sms) {
    double best = 1e30;
    int best_p = 1;
    for (int P = 1; P <= KC; ++P) {
        const int units = S * P;
        const int rounds = (units + sms - 1) / sms;
        const double load = rounds * (1.0 / P + 0.01);  // strips of bytes per CTA, plus epilogue
        if (load < best * 0.97) {
            best = load;
            best_p = P;
        }
    }
    return best_p;
}

constexpr int64_t kPairMinM = 256;  // below this the single-CTA tiles keep more SMs busy

}  // namespace

struct patch_group_s;

struct patch_handle_s {
    int device = 0;
    DeviceInfo dev;
    int64_t N = 0, K = 0;
    int R = 0, C = 0;
    Plan plan;
    uint8_t* packed = nullptr;
    uint32_t* slab_dev = nullptr;
    int* order_dev = nullptr;
    uint32_t* pgemm_dev = nullptr;  // the pair kernels' tables, rows in pair-position order
    uint32_t* pmeta_dev = nullptr;
    uint32_t* meta_dev = nullptr;
    uint32_t* gemm_dev = nullptr;
    int* status_dev = nullptr;
    int decode_parts = 1;                 // K-parts per strip for the decode kernel
    LinDesc desc{};                       // host copy of the device descriptor
    std::mutex groups_mu;
    std::vector<patch_group_s*> groups;   // groups this handle belongs to (its own one-member group too)
    CUtensorMap tm_a32, tm_a16, tm_a8, tm_e;
    patch_info_t info{};
    patch_group_s* self = nullptr;        // one-member group used by patch_linear
    std::mutex mu;
    void* stage_x = nullptr;
    size_t stage_x_bytes = 0;
    void* stage_y = nullptr;
    size_t stage_y_bytes = 0;
};

struct patch_group_s {
    int device = 0;
    DeviceInfo dev;
    int n = 0;
    patch_handle h[kMaxGroup] = {};
    int parts[kMaxGroup] = {};    // decode K-parts per strip of each member in this group
    int parts_w[kMaxGroup] = {};  // the same for the decode kernel's 64-token instance
    LinDesc* lins_dev = nullptr;  // n descriptors
    int* status_dev = nullptr;    // the first member's status word
    bool pure24 = false;          // every slab of every member runs on the sparse MMA
    std::mutex mu;
    std::mutex host_mu;           // serialises patch_group_linear_host calls on the host
    std::map<std::pair<int, int>, WorkList> work;  // (kernel, m_blocks or 0) -> schedule
    // decode workspaces: one per stream that issued an uncaptured decode call
    // (per thread for the per-thread default stream), and one that every
    // captured call bakes into its graph
    std::map<std::pair<cudaStream_t, size_t>, DecodeWs> decode_ws;
    DecodeWs capture_ws;
    // patch_group_linear_host: device staging (one X buffer per distinct
    // host input, one Y buffer per member), two copy streams, chunk events
    void* stage_x[kMaxGroup] = {};
    size_t stage_x_bytes[kMaxGroup] = {};
    void* stage_y[kMaxGroup] = {};
    size_t stage_y_bytes[kMaxGroup] = {};
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t last_done = nullptr;      // the previous host call's last copy back
    std::vector<cudaEvent_t> chunk_ev;    // 2 per chunk: inputs landed, outputs computed
};

namespace {

void free_ws(DecodeWs& w) {
    for (int i = 0; i < kMaxGroup; ++i) {
        cudaFree(w.partial[i]);
        cudaFree(w.partial_wide[i]);
        cudaFree(w.counters[i]);
        w.partial[i] = nullptr;
        w.partial_wide[i] = nullptr;
        w.counters[i] = nullptr;
    }
}

void free_group(patch_group g) {
    if (!g) return;
    cudaDeviceSynchronize();
    for (int i = 0; i < g->n; ++i) {
        if (!g->h[i]) continue;
        std::lock_guard<std::mutex> lk(g->h[i]->groups_mu);
        auto& v = g->h[i]->groups;
        v.erase(std::remove(v.begin(), v.end(), g), v.end());
    }
    cudaFree(g->lins_dev);
    for (auto& kv : g->work) {
        cudaFree(kv.second.off);
        cudaFree(kv.second.work);
        cudaFreeHost(kv.second.host);
        if (kv.second.ready) cudaEventDestroy(kv.second.ready);
    }
    for (auto& kv : g->decode_ws) free_ws(kv.second);
    free_ws(g->capture_ws);
    for (int i = 0; i < kMaxGroup; ++i) {
        cudaFree(g->stage_x[i]);
        cudaFree(g->stage_y[i]);
    }
    if (g->h2d) cudaStreamDestroy(g->h2d);
    if (g->d2h) cudaStreamDestroy(g->d2h);
    if (g->last_done) cudaEventDestroy(g->last_done);
    for (cudaEvent_t e : g->chunk_ev) cudaEventDestroy(e);
    delete g;
}

// Allocates a decode workspace for every member of g; counters zeroed on st.
patch_status alloc_ws(patch_group g, DecodeWs* w, cudaStream_t st) {
    for (int i = 0; i < g->n; ++i) {
        const int S = g->h[i]->plan.S, P = g->parts[i];
        w->S[i] = S;
        if ((P > 1 && cudaMalloc(&w->partial[i], sizeof(float) * (size_t)S * P * 128 * kDecodeBN) != cudaSuccess) ||
            cudaMalloc(&w->counters[i], sizeof(unsigned) * S) != cudaSuccess) {
            cudaGetLastError();
            free_ws(*w);
            return fail(PATCH_ERR_NOMEM, "decode workspace allocation failed");
        }
        cudaError_t e = cudaMemsetAsync(w->counters[i], 0, sizeof(unsigned) * S, st);
        if (e != cudaSuccess) {
            free_ws(*w);
            return cuda_fail(e, "decode workspace set-up");
        }
    }
    return PATCH_OK;
}

void free_handle(patch_handle h) {
    if (!h) return;
    cudaDeviceSynchronize();
    free_group(h->self);
    cudaFree(h->packed);
    cudaFree(h->slab_dev);
    cudaFree(h->order_dev);
    cudaFree(h->pgemm_dev);
    cudaFree(h->pmeta_dev);
    cudaFree(h->meta_dev);
    cudaFree(h->gemm_dev);
    cudaFree(h->status_dev);
    cudaFree(h->stage_x);
    cudaFree(h->stage_y);
    delete h;
}

patch_status make_group(const patch_handle* hs, int n, patch_group* out) {
    patch_group g = new (std::nothrow) patch_group_s();
    if (!g) return fail(PATCH_ERR_NOMEM, "host allocation failed");
    g->device = hs[0]->device;
    g->dev = hs[0]->dev;
    g->n = n;
    g->status_dev = hs[0]->status_dev;
    g->pure24 = true;
    for (int i = 0; i < n; ++i)
        g->pure24 = g->pure24 && hs[i]->plan.pair_sparse == (int64_t)hs[i]->plan.S * hs[i]->plan.KB;
    // the pure instance computes record offsets from the strip index, so it
    // also needs the pair order to be the strip order (always the case when
    // every slab is 2:4: all pairs then agree equally and the fixed ones stay)
    for (int i = 0; i < n && g->pure24; ++i)
        for (int q = 0; q < hs[i]->plan.S; ++q) g->pure24 = g->pure24 && hs[i]->plan.order[q] == q;
    LinDesc d[kMaxGroup];
    // Decode units: a lone linear keeps its own split (enough units for every
    // SM); in a group the members' units already fill the GPU, so parts are
    // made large (each unit's epilogue is then hidden behind streaming).
    double total = 0.0;
    for (int i = 0; i < n; ++i)
        for (double b : hs[i]->plan.strip_bytes) total += b;
    const double target = std::max(256.0 * 1024.0, total / (4.0 * kDecodeCtasPerSm * g->dev.sms));
    // the 64-token instance writes and sums four times the partial bytes per
    // part, so its parts are larger (a 4096-column strip is then one part;
    // on Llama-2-7B layers at M = 64, 78 % of HBM instead of 68 %)
    const double target_w =
        std::max(PATCH_DECODE_WIDE_PART_KB * 1024.0, total / (4.0 * kDecodeWideCtasPerSm * g->dev.sms));
    for (int i = 0; i < n; ++i) {
        g->h[i] = hs[i];
        d[i] = hs[i]->desc;
        int P = hs[i]->decode_parts, PW = P;
        if (n > 1) {
            const Plan& pl = hs[i]->plan;
            double avg = 0.0;
            for (double b : pl.strip_bytes) avg += b;
            avg /= std::max(1, pl.S);
            P = std::max(1, std::min(hs[i]->decode_parts, (int)(avg / target + 0.5)));
            PW = std::max(1, std::min(hs[i]->decode_parts, (int)(avg / target_w + 0.5)));
        }
        g->parts[i] = P;
        g->parts_w[i] = PW;
        d[i].P = P;
        d[i].PW = PW;
    }
    // Larger parts leave fewer units: keep them only while the group still
    // has about 2.5 units per SM (below that, SMs run one or two issue loops
    // and the stream slows more than the partial sums cost).
    int64_t units_w = 0;
    for (int i = 0; i < n; ++i) units_w += (int64_t)hs[i]->plan.S * g->parts_w[i];
    if (units_w * 2 < 5 * (int64_t)g->dev.sms)
        for (int i = 0; i < n; ++i) {
            g->parts_w[i] = g->parts[i];
            d[i].PW = d[i].P;
        }
    if (cudaMalloc(&g->lins_dev, sizeof(LinDesc) * n) != cudaSuccess) {
        cudaGetLastError();
        delete g;
        return fail(PATCH_ERR_NOMEM, "group descriptor allocation failed");
    }
    if (cudaMemcpy(g->lins_dev, d, sizeof(LinDesc) * n, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(g->lins_dev);
        delete g;
        return fail(PATCH_ERR_CUDA, "group descriptor upload failed");
    }
    patch_status st = alloc_ws(g, &g->capture_ws, nullptr);
    if (st == PATCH_OK && cudaDeviceSynchronize() != cudaSuccess) st = fail(PATCH_ERR_CUDA, "decode workspace set-up");
    if (st != PATCH_OK) {
        cudaFree(g->lins_dev);
        delete g;
        return st;
    }
    for (int i = 0; i < n; ++i) {
        std::lock_guard<std::mutex> lk(hs[i]->groups_mu);
        hs[i]->groups.push_back(g);
    }
    *out = g;
    return PATCH_OK;
}

// Gives w the 64-token partial buffers if it lacks them (once; they live
// until the group is destroyed, so captured graphs may keep their address).
patch_status ensure_wide_ws(patch_group g, DecodeWs* w) {
    for (int i = 0; i < g->n; ++i) {
        if (g->parts_w[i] <= 1 || w->partial_wide[i]) continue;
        if (cudaMalloc(&w->partial_wide[i], sizeof(float) * (size_t)w->S[i] * g->parts_w[i] * 128 * kDecodeWideBN) !=
            cudaSuccess) {
            cudaGetLastError();
            w->partial_wide[i] = nullptr;
            return fail(PATCH_ERR_NOMEM, "decode workspace allocation failed");
        }
    }
    return PATCH_OK;
}

// The decode workspace a call on `st` uses: the capture workspace when the
// stream is capturing a graph, else the stream's own (allocated on its first
// decode call; for the per-thread default stream, one per thread). A call
// with bn = kDecodeWideBN also gives the capture workspace its 64-token
// buffers, so a graph captured after one uncaptured call of that size
// allocates nothing.
patch_status get_decode_ws(patch_group g, cudaStream_t st, int bn, const DecodeWs** out) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    const bool wide = bn == kDecodeWideBN;
    std::lock_guard<std::mutex> lk(g->mu);
    if (wide) {
        patch_status s = ensure_wide_ws(g, &g->capture_ws);
        if (s != PATCH_OK) return s;
    }
    if (cs != cudaStreamCaptureStatusNone) {
        *out = &g->capture_ws;
        return PATCH_OK;
    }
    const size_t tid = st == cudaStreamPerThread ? std::hash<std::thread::id>()(std::this_thread::get_id()) : 0;
    const auto key = std::make_pair(st, tid);
    auto it = g->decode_ws.find(key);
    if (it == g->decode_ws.end()) {
        DecodeWs w;
        patch_status s = alloc_ws(g, &w, st);
        if (s != PATCH_OK) return s;
        it = g->decode_ws.emplace(key, w).first;
    }
    if (wide) {
        patch_status s = ensure_wide_ws(g, &it->second);
        if (s != PATCH_OK) return s;
    }
    *out = &it->second;
    return PATCH_OK;
}

// Greedy longest-processing-time assignment of the group's units to
// persistent CTAs (or clusters). kernel 0: (strip, token block), cost = slab
// work (dense 1, 2:4 1/2) + one epilogue; kernel 1: (strip pair, token block),
// same costs; kernel 3: (four strips, token block), the slower pair's cost;
// kernels 2 and 5: (strip, K-part), cost = streamed bytes of the part.
// Per tensor-core kernel (0 single CTA, 1 CTA pair, 2 decode with 16-token
// MMAs, 4 CTA pair with two strips per CTA, 5 decode with 64-token MMAs):
// tokens per tile,
// activation rows per TMA box, weight rows of a work unit, persistent slots.
int kernel_bn(int kernel) {
    return kernel == 0   ? kGemmBN
           : kernel == 2 ? kDecodeBN
           : kernel == 5 ? kDecodeWideBN
           : kernel == 4 ? kGemm22BN
                         : kGemm2BN;
}
int kernel_box_rows(int kernel) {
    return kernel == 1 ? kGemm2BN / 2 : kernel == 4 ? kGemm22BN / 2 : kernel_bn(kernel);
}
int64_t kernel_rows(const Plan& p, int kernel) {
    const int64_t pairs = (int64_t)p.pair_cost.size();
    return kernel == 0 ? (int64_t)p.strip_cost.size() : kernel == 1 ? pairs : (pairs + 1) / 2;
}
int kernel_slots(const DeviceInfo& d, int kernel) {
    return kernel == 1   ? d.pair_clusters
           : kernel == 4 ? d.wide_clusters
           : kernel == 2 ? kDecodeCtasPerSm * d.sms
           : kernel == 5 ? kDecodeWideCtasPerSm * d.sms
                         : d.sms;
}

void lpt_schedule(patch_group g, int kernel, int mb, std::vector<int>& off, std::vector<int>& work) {
    struct Unit {
        double cost;
        int id;
    };
    std::vector<Unit> units;
    for (int l = 0; l < g->n; ++l) {
        const Plan& p = g->h[l]->plan;
        if (kernel == 0 || kernel == 1) {
            const std::vector<double>& c = kernel == 0 ? p.strip_cost : p.pair_cost;
            for (int r = 0; r < (int)c.size(); ++r)
                for (int j = 0; j < mb; ++j) units.push_back({c[r] + 1.0, (l << kUnitShift) | (r * mb + j)});
        } else if (kernel == 4) {
            // a strip quad issues both of its pairs' MMAs at every slab
            const std::vector<double>& c = p.pair_cost;
            for (int r = 0; r < (int)(c.size() + 1) / 2; ++r) {
                const double cost = c[2 * r] + (2 * r + 1 < (int)c.size() ? c[2 * r + 1] : c[2 * r]);
                for (int j = 0; j < mb; ++j) units.push_back({cost + 2.0, (l << kUnitShift) | (r * mb + j)});
            }
        } else {
            const int P = kernel == 5 ? g->parts_w[l] : g->parts[l];
            for (int s = 0; s < p.S; ++s)
                for (int q = 0; q < P; ++q)
                    units.push_back({p.strip_bytes[s] / P + 16384.0, (l << kUnitShift) | (s * P + q)});
        }
    }
    std::stable_sort(units.begin(), units.end(), [](const Unit& x, const Unit& y) { return x.cost > y.cost; });
    const int grid = std::max(1, std::min(kernel_slots(g->dev, kernel), (int)units.size()));
    using Item = std::pair<double, int>;
    std::priority_queue<Item, std::vector<Item>, std::greater<Item>> pq;
    for (int c = 0; c < grid; ++c) pq.push({0.0, c});
    std::vector<std::vector<int>> lists(grid);
    for (const Unit& u : units) {
        Item top = pq.top();
        pq.pop();
        lists[top.second].push_back(u.id);
        top.first += u.cost;
        pq.push(top);
    }
    off.assign(grid + 1, 0);
    work.clear();
    for (int c = 0; c < grid; ++c) {
        off[c] = (int)work.size();
        work.insert(work.end(), lists[c].begin(), lists[c].end());
    }
    off[grid] = (int)work.size();
}

// The cached schedule of (kernel, mb). The first call for a key builds it and
// uploads it asynchronously on `st` from a pinned host copy; a call on another
// stream waits for that upload through an event until it is known complete.
patch_status get_worklist(patch_group g, int kernel, int mb, cudaStream_t st, WorkList** out) {
    WorkList* wl = nullptr;
    {
        std::lock_guard<std::mutex> lk(g->mu);
        auto key = std::make_pair(kernel, mb);
        auto it = g->work.find(key);
        if (it == g->work.end()) {
            std::vector<int> off, work;
            lpt_schedule(g, kernel, mb, off, work);
            const size_t n_off = off.size(), n_work = std::max<size_t>(work.size(), 1);
            int *d_off = nullptr, *d_work = nullptr, *host = nullptr;
            cudaEvent_t ev = nullptr;
            if (cudaMalloc(&d_off, sizeof(int) * n_off) != cudaSuccess ||
                cudaMalloc(&d_work, sizeof(int) * n_work) != cudaSuccess ||
                cudaHostAlloc(&host, sizeof(int) * (n_off + n_work), cudaHostAllocDefault) != cudaSuccess ||
                cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
                cudaGetLastError();
                cudaFree(d_off);
                cudaFree(d_work);
                cudaFreeHost(host);
                return fail(PATCH_ERR_NOMEM, "schedule allocation failed");
            }
            std::copy(off.begin(), off.end(), host);
            std::copy(work.begin(), work.end(), host + n_off);
            cudaError_t e = cudaMemcpyAsync(d_off, host, sizeof(int) * n_off, cudaMemcpyHostToDevice, st);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(d_work, host + n_off, sizeof(int) * work.size(), cudaMemcpyHostToDevice, st);
            if (e == cudaSuccess) e = cudaEventRecord(ev, st);
            it = g->work.emplace(std::piecewise_construct, std::forward_as_tuple(key), std::forward_as_tuple()).first;
            WorkList& w = it->second;
            w.grid = (int)n_off - 1;
            w.off = d_off;
            w.work = d_work;
            w.host = host;
            w.ready = ev;
            w.made_on = st;
            if (e != cudaSuccess) {
                // keep nothing half-built: later calls must rebuild it
                cudaStreamSynchronize(st);
                cudaFree(d_off);
                cudaFree(d_work);
                cudaFreeHost(host);
                cudaEventDestroy(ev);
                g->work.erase(it);
                return cuda_fail(e, "schedule upload");
            }
            *out = &w;
            return PATCH_OK;
        }
        wl = &it->second;
    }
    if (!wl->done.load(std::memory_order_acquire) && st != wl->made_on) {
        // a stream that is capturing a graph makes no event call: the first
        // call for this M has completed before capture (documented rule)
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        PATCH_CUDA(cudaStreamIsCapturing(st, &cs));
        if (cs != cudaStreamCaptureStatusNone) {
            *out = wl;
            return PATCH_OK;
        }
        const cudaError_t q = cudaEventQuery(wl->ready);
        if (q == cudaSuccess) {
            wl->done.store(true, std::memory_order_release);
        } else if (q == cudaErrorNotReady) {
            PATCH_CUDA(cudaStreamWaitEvent(st, wl->ready, 0));
        } else {
            return cuda_fail(q, "schedule upload");
        }
    }
    *out = wl;
    return PATCH_OK;
}

patch_status check_device_is(int device) {
    int dev = -1;
    PATCH_CUDA(cudaGetDevice(&dev));
    if (dev != device) return fail(PATCH_ERR_ARG, "handle lives on device %d, current device is %d", device, dev);
    return PATCH_OK;
}

// Resolves AUTO / GEMM to a concrete kernel for this M.
// AUTO and GEMM pick by M; for large M the two-strips-per-CTA kernel is used
// when the launch has enough strip quads to keep every CTA pair busy (it
// feeds each activation tile to twice the weight rows, but a small weight
// gives it half as many work units as the one-strip pair kernel).
// The wide kernel runs its pure 2:4 instance (GEMM_WIDE_24) when every slab
// of every member runs on the sparse MMA.
int resolve_path(patch_group g, int path, int64_t M) {
    if (path == PATCH_PATH_AUTO) path = (M <= kDecodeWideBN) ? PATCH_PATH_GEMV : PATCH_PATH_GEMM;
    if (path == PATCH_PATH_GEMM) {
        if (M < kPairMinM) return PATCH_PATH_GEMM_SINGLE;
        int64_t quads = 0;
        for (int l = 0; l < g->n; ++l) quads += (g->h[l]->plan.S + 3) / 4;
        const int64_t units = quads * ((M + kGemm22BN - 1) / kGemm22BN);
        path = units >= 2 * (int64_t)g->dev.wide_clusters ? PATCH_PATH_GEMM_WIDE : PATCH_PATH_GEMM_PAIR;
    }
    if (path == PATCH_PATH_GEMM_WIDE && g->pure24) return PATCH_PATH_GEMM_WIDE_24;
    return path;
}

patch_status run_simt(patch_handle h, const void* X, int64_t M, void* Y, cudaStream_t st) {
    if (M > 16) return fail(PATCH_ERR_SHAPE, "the CUDA-core decode kernel takes M <= 16 (got %lld)", (long long)M);
    GemvArgs a;
    a.packed = h->packed;
    a.slab = h->slab_dev;
    a.meta = h->meta_dev;
    a.X = static_cast<const __nv_bfloat16*>(X);
    a.Y = static_cast<__nv_bfloat16*>(Y);
    a.M = (int)M;
    a.N = (int)h->N;
    a.K = (int)h->K;
    a.KB = h->plan.KB;
    a.KC = h->plan.KC;
    cudaError_t e = launch_gemv(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "CUDA-core decode kernel launch");
    return PATCH_OK;
}

// Kernel for a resolved path: 0 single CTA, 1 CTA pair, 4 CTA pair with two
// strips per CTA, 2 / 5 decode with 16- / 64-token MMAs.
int choose_kernel(patch_group g, int path, int64_t M) {
    (void)g;
    if (path == PATCH_PATH_GEMM_SINGLE) return 0;
    if (path == PATCH_PATH_GEMV) return M <= kDecodeBN ? 2 : 5;
    if (path == PATCH_PATH_GEMM_WIDE || path == PATCH_PATH_GEMM_WIDE_24) return 4;
    return 1;
}

// One launch over every member of the group. `sched` (off, work) may point at
// caller-provided device memory; otherwise the group's cached schedule is used.
patch_status run_group(patch_group g, const void* const* X, int64_t M, void* const* Y, int path, cudaStream_t st,
                       const int* sched_off = nullptr, const int* sched_work = nullptr, int sched_grid = 0) {
    path = resolve_path(g, path, M);
    if (path == PATCH_PATH_GEMV_SIMT) {
        for (int l = 0; l < g->n; ++l) {
            patch_status s = run_simt(g->h[l], X[l], M, Y[l], st);
            if (s != PATCH_OK) return s;
        }
        return PATCH_OK;
    }
    if (path != PATCH_PATH_GEMV && path != PATCH_PATH_GEMM_SINGLE && path != PATCH_PATH_GEMM_PAIR &&
        path != PATCH_PATH_GEMM_WIDE && path != PATCH_PATH_GEMM_WIDE_24)
        return fail(PATCH_ERR_ARG, "unknown path %d", path);
    if (path == PATCH_PATH_GEMM_WIDE_24 && !g->pure24)
        return fail(PATCH_ERR_ARG, "GEMM_WIDE_24 needs every slab of every member to be 2:4 in both strips of its pair");
    if (path == PATCH_PATH_GEMV && M > kDecodeWideBN)
        return fail(PATCH_ERR_SHAPE, "the decode kernel takes M <= %d (got %lld)", kDecodeWideBN, (long long)M);
    if (M > (int64_t)INT32_MAX / 2) return fail(PATCH_ERR_SHAPE, "M too large");
    const int kernel = choose_kernel(g, path, M);
    const bool decode = kernel == 2 || kernel == 5;
    const int bn = kernel_bn(kernel);
    const int mb = decode ? 0 : (int)((M + bn - 1) / bn);
    // the decode kernels load (and multiply) only M rounded up to 16 tokens
    const int box_rows = decode ? (int)std::min<int64_t>(bn, (M + 15) & ~15) : kernel_box_rows(kernel);
    GroupMaps maps;
    GroupArgs a;
    memset(&maps, 0, sizeof(maps));
    memset(&a, 0, sizeof(a));
    for (int l = 0; l < g->n; ++l) {
        patch_handle h = g->h[l];
        patch_status s = encode_2d(&maps.x[l], X[l], h->K, M, kSlabK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
        if (s != PATCH_OK) return s;
        maps.a32[l] = h->tm_a32;
        maps.a16[l] = h->tm_a16;
        maps.a8[l] = h->tm_a8;
        maps.e[l] = h->tm_e;
        a.Y[l] = static_cast<__nv_bfloat16*>(Y[l]);
    }
    int grid = sched_grid;
    if (!sched_off) {
        WorkList* wl = nullptr;
        patch_status s = get_worklist(g, kernel, mb, st, &wl);
        if (s != PATCH_OK) return s;
        sched_off = wl->off;
        sched_work = wl->work;
        grid = wl->grid;
    }
    if (decode) {
        const DecodeWs* ws = nullptr;
        patch_status s = get_decode_ws(g, st, bn, &ws);
        if (s != PATCH_OK) return s;
        for (int l = 0; l < g->n; ++l) {
            a.partial[l] = kernel == 5 ? ws->partial_wide[l] : ws->partial[l];
            a.counters[l] = ws->counters[l];
        }
    }
    a.lins = g->lins_dev;
    a.work_off = sched_off;
    a.work = sched_work;
    a.M = (int)M;
    a.MB = mb;
    if (mb > 0) {
        const int64_t gran = (M + 15) / 16;
        a.tile_gran = (int)(gran / mb);
        a.tile_extra = (int)(gran % mb);
    }
    a.status = g->status_dev;
    cudaError_t e = kernel == 0   ? launch_gemm(maps, a, grid, st)
                    : kernel == 1 ? launch_gemm2(maps, a, grid, st)
                    : kernel == 4 ? launch_gemm22(maps, a, grid, path == PATCH_PATH_GEMM_WIDE_24, st)
                                  : launch_decode(maps, a, grid, bn, st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel launch");
    return PATCH_OK;
}

patch_status check_xy(const void* X, const void* Y) {
    if (!X || !Y) return fail(PATCH_ERR_ARG, "X and Y must be non-NULL");
    if (!aligned16(X) || !aligned16(Y)) return fail(PATCH_ERR_ALIGN, "X and Y must be 16-byte aligned");
    return PATCH_OK;
}

}  // namespace

extern "C" {

const char* patch_last_error(void) { return g_err.c_str(); }

int patch_version(void) { return 4; }

patch_status patch_plan(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows, int tile_cols,
                        uint32_t* slab_table, uint32_t* meta_table, uint32_t* gemm_table, int64_t* packed_bytes) {
    if (!tile_flags) return fail(PATCH_ERR_ARG, "tile_flags is NULL");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    st = check_flags(tile_flags, (N / tile_rows) * (K / tile_cols));
    if (st != PATCH_OK) return st;
    Plan p;
    build_plan(p, N, K, tile_rows, tile_cols, tile_flags);
    if (slab_table) memcpy(slab_table, p.slab.data(), sizeof(uint32_t) * p.slab.size());
    if (meta_table) memcpy(meta_table, p.meta.data(), sizeof(uint32_t) * p.meta.size());
    if (gemm_table) memcpy(gemm_table, p.gemm.data(), sizeof(uint32_t) * p.gemm.size());
    if (packed_bytes) *packed_bytes = p.bytes;
    return PATCH_OK;
}

patch_status patch_plan_pairs(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows, int tile_cols,
                              int32_t* order) {
    if (!tile_flags || !order) return fail(PATCH_ERR_ARG, "tile_flags and order must be non-NULL");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    st = check_flags(tile_flags, (N / tile_rows) * (K / tile_cols));
    if (st != PATCH_OK) return st;
    Plan p;
    build_plan(p, N, K, tile_rows, tile_cols, tile_flags);
    for (int q = 0; q < p.S; ++q) order[q] = p.order[q];
    return PATCH_OK;
}

patch_status patch_classify_tiles(const uint8_t* mask_bits, int64_t N, int64_t K, int tile_rows, int tile_cols,
                                  uint8_t* tile_flags, int64_t* dense_with_pruned) {
    if (!mask_bits || !tile_flags) return fail(PATCH_ERR_ARG, "mask_bits and tile_flags must be non-NULL");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    // K and the tile width are multiples of 8, so every mask byte holds two
    // whole groups of four k (one per nibble) in either bit order.
    auto two_of_four = [](unsigned v) { return __builtin_popcount(v) == 2; };
    const int64_t tiles_k = K / tile_cols, row_bytes = K / 8, tile_bytes = tile_cols / 8;
    int64_t stray = 0;
    for (int64_t tr = 0; tr < N / tile_rows; ++tr)
        for (int64_t tc = 0; tc < tiles_k; ++tc) {
            bool sparse = true, full = true;
            for (int64_t r = tr * tile_rows; r < (tr + 1) * tile_rows; ++r) {
                const uint8_t* row = mask_bits + r * row_bytes + tc * tile_bytes;
                for (int64_t i = 0; i < tile_bytes; ++i) {
                    sparse = sparse && two_of_four(row[i] >> 4) && two_of_four(row[i] & 15u);
                    full = full && row[i] == 0xFF;
                }
            }
            tile_flags[tr * tiles_k + tc] = sparse ? 1 : 0;
            stray += !sparse && !full;
        }
    if (dense_with_pruned) *dense_with_pruned = stray;
    return PATCH_OK;
}

patch_status patch_partition_rows(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows, int tile_cols,
                                  int parts, int64_t align_rows, int64_t* bounds) {
    if (!tile_flags || !bounds) return fail(PATCH_ERR_ARG, "tile_flags and bounds must be non-NULL");
    if (parts < 1) return fail(PATCH_ERR_ARG, "parts must be at least 1");
    if (align_rows <= 0 || align_rows % (2 * kStrip) != 0)
        return fail(PATCH_ERR_ARG, "align_rows must be a positive multiple of 256");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    st = check_flags(tile_flags, (N / tile_rows) * (K / tile_cols));
    if (st != PATCH_OK) return st;
    Plan p;
    build_plan(p, N, K, tile_rows, tile_cols, tile_flags);
    // Unit u = align_rows / 256 consecutive strip pairs. Its cost, in half
    // dense slabs so that it is an integer: every slab of a pair (dense 2,
    // paired 2:4 1) plus 2 for the pair's epilogue, as the tile scheduler counts.
    const int64_t per_unit = align_rows / (2 * kStrip);
    const int64_t pairs = (int64_t)p.pair_cost.size();
    const int64_t units = (pairs + per_unit - 1) / per_unit;
    std::vector<int64_t> cost((size_t)units, 0);
    for (int64_t q = 0; q < pairs; ++q) cost[(size_t)(q / per_unit)] += (int64_t)llround(2.0 * p.adj_pair_cost[q]) + 2;
    // Smallest bottleneck T that a left-to-right greedy packing fits into
    // `parts` contiguous parts (the greedy is optimal for a given T).
    auto parts_needed = [&](int64_t T) {
        int64_t n = 1, acc = 0;
        for (int64_t c : cost) {
            if (acc + c > T) {
                ++n;
                acc = c;
            } else {
                acc += c;
            }
        }
        return n;
    };
    int64_t lo = 0, hi = 0;
    for (int64_t c : cost) {
        lo = std::max(lo, c);
        hi += c;
    }
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (parts_needed(mid) <= parts)
            hi = mid;
        else
            lo = mid + 1;
    }
    // Lay the parts out under T = lo, stopping a part early only to leave
    // one unit for every later part, so no rank idles while units remain.
    int64_t u = 0;
    bounds[0] = 0;
    for (int r = 0; r < parts; ++r) {
        const int64_t later = parts - 1 - r;
        int64_t acc = 0;
        while (u < units && acc + cost[(size_t)u] <= lo && (acc == 0 || units - u - 1 >= later)) {
            acc += cost[(size_t)u];
            ++u;
        }
        bounds[r + 1] = std::min<int64_t>(N, u * align_rows);
    }
    if (u != units) return fail(PATCH_ERR_ARG, "internal: partition left rows unassigned");
    return PATCH_OK;
}

patch_status patch_pack(const void* W_bf16, int64_t N, int64_t K, const uint8_t* mask_bits, int bitorder,
                        const uint8_t* tile_flags, int tile_rows, int tile_cols, void* stream,
                        patch_handle* out) {
    if (!out) return fail(PATCH_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (!W_bf16 || !mask_bits || !tile_flags)
        return fail(PATCH_ERR_ARG, "W, mask_bits and tile_flags must be non-NULL");
    if (bitorder != 0 && bitorder != 1) return fail(PATCH_ERR_ARG, "bitorder must be 0 or 1");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    if (!aligned16(W_bf16)) return fail(PATCH_ERR_ALIGN, "W must be 16-byte aligned");
    const int64_t ntiles = (N / tile_rows) * (K / tile_cols);
    st = check_flags(tile_flags, ntiles);
    if (st != PATCH_OK) return st;
    int dev = 0;
    DeviceInfo di;
    st = prepare_device(&dev, &di);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    patch_handle h = new (std::nothrow) patch_handle_s();
    if (!h) return fail(PATCH_ERR_NOMEM, "host allocation failed");
    h->device = dev;
    h->dev = di;
    h->N = N;
    h->K = K;
    h->R = tile_rows;
    h->C = tile_cols;
    build_plan(h->plan, N, K, tile_rows, tile_cols, tile_flags);
    const Plan& p = h->plan;
    if (p.bytes / 16 >= ((int64_t)1 << 30)) {
        free_handle(h);
        return fail(PATCH_ERR_SHAPE, "packed weight exceeds the 16 GiB table range");
    }
    int64_t tiles_sparse = 0;
    for (int64_t i = 0; i < ntiles; ++i) tiles_sparse += tile_flags[i];
    h->decode_parts = choose_decode_parts(p.S, p.KC, kDecodeCtasPerSm * di.sms);

    uint8_t* flags_dev = nullptr;
    unsigned long long* counters = nullptr;
    auto cleanup = [&](patch_status code) {
        cudaFree(flags_dev);
        cudaFree(counters);
        if (code != PATCH_OK) free_handle(h);
        return code;
    };
    if (cudaMalloc(&h->packed, std::max<int64_t>(p.bytes, 2048)) != cudaSuccess ||
        cudaMalloc(&h->slab_dev, sizeof(uint32_t) * p.slab.size()) != cudaSuccess ||
        cudaMalloc(&h->order_dev, sizeof(int) * p.order.size()) != cudaSuccess ||
        cudaMalloc(&h->pgemm_dev, sizeof(uint32_t) * p.pgemm.size()) != cudaSuccess ||
        cudaMalloc(&h->pmeta_dev, sizeof(uint32_t) * p.pmeta.size()) != cudaSuccess ||
        cudaMalloc(&h->meta_dev, sizeof(uint32_t) * p.meta.size()) != cudaSuccess ||
        cudaMalloc(&h->gemm_dev, sizeof(uint32_t) * p.gemm.size()) != cudaSuccess ||
        cudaMalloc(&h->status_dev, sizeof(int)) != cudaSuccess ||
        cudaMalloc(&flags_dev, ntiles) != cudaSuccess ||
        cudaMalloc(&counters, 3 * sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        return cleanup(fail(PATCH_ERR_NOMEM, "device allocation of %lld packed bytes failed", (long long)p.bytes));
    }
    // tensor maps of the packed bytes viewed as rows of 64 bf16 (128 bytes):
    // two adjacent dense records (256 rows), a dense slab / dense image or two
    // adjacent 2:4 records (128 rows), 2:4 values (64 rows), metadata (16 rows)
    const int64_t rows = std::max<int64_t>(p.bytes, 2048) / 128;
    if ((st = encode_2d(&h->tm_a32, h->packed, 64, rows, 64, 256, CU_TENSOR_MAP_SWIZZLE_NONE)) != PATCH_OK ||
        (st = encode_2d(&h->tm_a16, h->packed, 64, rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE)) != PATCH_OK ||
        (st = encode_2d(&h->tm_a8, h->packed, 64, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE)) != PATCH_OK ||
        (st = encode_2d(&h->tm_e, h->packed, 64, rows, 64, 16, CU_TENSOR_MAP_SWIZZLE_NONE)) != PATCH_OK)
        return cleanup(st);
    cudaError_t e;
    if ((e = cudaMemcpyAsync(h->slab_dev, p.slab.data(), sizeof(uint32_t) * p.slab.size(), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h->meta_dev, p.meta.data(), sizeof(uint32_t) * p.meta.size(), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h->gemm_dev, p.gemm.data(), sizeof(uint32_t) * p.gemm.size(), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h->order_dev, p.order.data(), sizeof(int) * p.order.size(), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h->pgemm_dev, p.pgemm.data(), sizeof(uint32_t) * p.pgemm.size(),
                             cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h->pmeta_dev, p.pmeta.data(), sizeof(uint32_t) * p.pmeta.size(),
                             cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(flags_dev, tile_flags, ntiles, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(counters, 0, 3 * sizeof(unsigned long long), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(h->status_dev, 0, sizeof(int), s)) != cudaSuccess)
        return cleanup(cuda_fail(e, "pack set-up copies"));
    PackArgs a;
    a.W = static_cast<const uint16_t*>(W_bf16);
    a.bits = mask_bits;
    a.bitorder = bitorder;
    a.flags = flags_dev;
    a.slab = h->slab_dev;
    a.meta = h->meta_dev;
    a.gemm = h->gemm_dev;
    a.out = h->packed;
    a.K = K;
    a.R = tile_rows;
    a.C = tile_cols;
    a.KB = p.KB;
    a.KC = p.KC;
    a.counters = counters;
    pack_kernel<<<p.S * p.KB, 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return cleanup(cuda_fail(e, "pack kernel launch"));
    unsigned long long cnt[3] = {0, 0, 0};
    if ((e = cudaMemcpyAsync(cnt, counters, sizeof(cnt), cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
        return cleanup(cuda_fail(e, "pack kernel"));
    if (cnt[0] != 0)
        return cleanup(fail(PATCH_ERR_MASK, "%llu groups inside 2:4 tiles do not keep exactly two of four", cnt[0]));
    h->desc.packed = h->packed;
    h->desc.slab = h->slab_dev;
    h->desc.meta = h->meta_dev;
    h->desc.gemm = h->pgemm_dev;
    h->desc.pmeta = h->pmeta_dev;
    h->desc.order = h->order_dev;
    h->desc.N = (int)N;
    h->desc.S = p.S;
    h->desc.KB = p.KB;
    h->desc.KC = p.KC;
    h->desc.P = h->decode_parts;
    h->desc.PW = h->decode_parts;
    patch_handle self[1] = {h};
    if ((st = make_group(self, 1, &h->self)) != PATCH_OK) return cleanup(st);
    patch_info_t& info = h->info;
    info.N = N;
    info.K = K;
    info.tile_rows = tile_rows;
    info.tile_cols = tile_cols;
    info.tiles_total = ntiles;
    info.tiles_sparse = tiles_sparse;
    info.slabs_total = (int64_t)p.S * p.KB;
    info.slabs_sparse = p.sparse;
    info.slabs_pair_sparse = p.pair_sparse;
    info.meta_blocks = p.meta_blocks;
    info.dense_images = p.images;
    info.packed_bytes = p.bytes;
    info.pruned = (int64_t)cnt[2];
    info.stray_zeros = (int64_t)cnt[1];
    info.sparsity = (double)cnt[2] / (double)(N * K);
    *out = h;
    return cleanup(PATCH_OK);
}

patch_status patch_linear_path(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16, int path,
                               void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (path < PATCH_PATH_AUTO || path > PATCH_PATH_GEMM_WIDE_24) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    if (M == 0) return PATCH_OK;
    patch_status st = check_xy(X_bf16, Y_bf16);
    if (st != PATCH_OK) return st;
    if ((st = check_device_is(h->device)) != PATCH_OK) return st;
    const void* xs[1] = {X_bf16};
    void* ys[1] = {Y_bf16};
    return run_group(h->self, xs, M, ys, path, static_cast<cudaStream_t>(stream));
}

patch_status patch_linear(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16, void* stream) {
    return patch_linear_path(h, X_bf16, M, Y_bf16, PATCH_PATH_AUTO, stream);
}

patch_status patch_linear_host(patch_handle h, const void* X_host, int64_t M, void* Y_host, void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (M == 0) return PATCH_OK;
    if (!X_host || !Y_host) return fail(PATCH_ERR_ARG, "X and Y must be non-NULL");
    patch_status st = check_device_is(h->device);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lk(h->mu);
    const size_t xb = (size_t)M * h->K * 2, yb = (size_t)M * h->N * 2;
    if (xb > h->stage_x_bytes) {
        cudaFree(h->stage_x);
        h->stage_x = nullptr;
        h->stage_x_bytes = 0;
        if (cudaMalloc(&h->stage_x, xb) != cudaSuccess) {
            cudaGetLastError();
            return fail(PATCH_ERR_NOMEM, "staging allocation failed");
        }
        h->stage_x_bytes = xb;
    }
    if (yb > h->stage_y_bytes) {
        cudaFree(h->stage_y);
        h->stage_y = nullptr;
        h->stage_y_bytes = 0;
        if (cudaMalloc(&h->stage_y, yb) != cudaSuccess) {
            cudaGetLastError();
            return fail(PATCH_ERR_NOMEM, "staging allocation failed");
        }
        h->stage_y_bytes = yb;
    }
    PATCH_CUDA(cudaMemcpyAsync(h->stage_x, X_host, xb, cudaMemcpyHostToDevice, s));
    const void* xs[1] = {h->stage_x};
    void* ys[1] = {h->stage_y};
    st = run_group(h->self, xs, M, ys, PATCH_PATH_AUTO, s);
    if (st != PATCH_OK) return st;
    PATCH_CUDA(cudaMemcpyAsync(Y_host, h->stage_y, yb, cudaMemcpyDeviceToHost, s));
    PATCH_CUDA(cudaStreamSynchronize(s));
    return PATCH_OK;
}

patch_status patch_group_create(const patch_handle* handles, int n, patch_group* out) {
    if (!out) return fail(PATCH_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (!handles || n < 1 || n > kMaxGroup) return fail(PATCH_ERR_ARG, "a group takes 1 to %d handles", kMaxGroup);
    for (int i = 0; i < n; ++i) {
        if (!handles[i]) return fail(PATCH_ERR_ARG, "handle %d is NULL", i);
        if (handles[i]->device != handles[0]->device) return fail(PATCH_ERR_ARG, "handles live on different devices");
    }
    patch_status st = check_device_is(handles[0]->device);
    if (st != PATCH_OK) return st;
    return make_group(handles, n, out);
}

patch_status patch_group_linear(patch_group g, const void* const* X, int64_t M, void* const* Y, int path,
                                void* stream) {
    if (!g) return fail(PATCH_ERR_ARG, "group is NULL");
    if (!X || !Y) return fail(PATCH_ERR_ARG, "X and Y arrays must be non-NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (path < PATCH_PATH_AUTO || path > PATCH_PATH_GEMM_WIDE_24) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    if (M == 0) return PATCH_OK;
    for (int l = 0; l < g->n; ++l) {
        patch_status st = check_xy(X[l], Y[l]);
        if (st != PATCH_OK) return st;
    }
    patch_status st = check_device_is(g->device);
    if (st != PATCH_OK) return st;
    return run_group(g, X, M, Y, path, static_cast<cudaStream_t>(stream));
}

patch_status patch_group_path(patch_group g, int64_t M, int path, int* out) {
    if (!g || !out) return fail(PATCH_ERR_ARG, "group and out must be non-NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (path < PATCH_PATH_AUTO || path > PATCH_PATH_GEMM_WIDE_24) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    *out = resolve_path(g, path, M);
    return PATCH_OK;
}

void patch_group_free(patch_group g) { free_group(g); }

patch_status patch_group_linear_host(patch_group g, const void* const* X_host, int64_t M, void* const* Y_host,
                                     int path, void* stream) {
    if (!g) return fail(PATCH_ERR_ARG, "group is NULL");
    if (!X_host || !Y_host) return fail(PATCH_ERR_ARG, "X and Y arrays must be non-NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (path < PATCH_PATH_AUTO || path > PATCH_PATH_GEMM_WIDE_24) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    for (int l = 0; l < g->n; ++l)
        if (!X_host[l] || !Y_host[l]) return fail(PATCH_ERR_ARG, "member %d: X and Y must be non-NULL", l);
    if (M == 0) return PATCH_OK;
    if (M > (int64_t)INT32_MAX / 2) return fail(PATCH_ERR_SHAPE, "M too large");
    patch_status st = check_device_is(g->device);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lk(g->host_mu);

    // distinct inputs (q, k, v read one X): slot of each member
    int slot[kMaxGroup], nslots = 0;
    const void* src[kMaxGroup];
    int64_t slotK[kMaxGroup];
    for (int l = 0; l < g->n; ++l) {
        int f = -1;
        for (int i = 0; i < nslots; ++i)
            if (src[i] == X_host[l] && slotK[i] == g->h[l]->K) f = i;
        if (f < 0) {
            f = nslots++;
            src[f] = X_host[l];
            slotK[f] = g->h[l]->K;
        }
        slot[l] = f;
    }
    auto grow = [&](void** buf, size_t* have, size_t need) {
        if (need <= *have) return true;
        cudaFree(*buf);
        *buf = nullptr;
        *have = 0;
        if (cudaMalloc(buf, need) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        *have = need;
        return true;
    };
    if (!g->h2d) {
        if (cudaStreamCreateWithFlags(&g->h2d, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&g->d2h, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&g->last_done, cudaEventDisableTiming) != cudaSuccess)
            return fail(PATCH_ERR_CUDA, "copy stream set-up failed");
        PATCH_CUDA(cudaEventRecord(g->last_done, g->d2h));
    }
    // The previous host call on this group must be done with the staging
    // buffers before they are regrown or overwritten.
    bool regrow = false;
    for (int i = 0; i < nslots; ++i) regrow = regrow || (size_t)M * slotK[i] * 2 > g->stage_x_bytes[i];
    for (int l = 0; l < g->n; ++l) regrow = regrow || (size_t)M * g->h[l]->N * 2 > g->stage_y_bytes[l];
    if (regrow) PATCH_CUDA(cudaEventSynchronize(g->last_done));
    for (int i = 0; i < nslots; ++i)
        if (!grow(&g->stage_x[i], &g->stage_x_bytes[i], (size_t)M * slotK[i] * 2))
            return fail(PATCH_ERR_NOMEM, "staging allocation failed");
    for (int l = 0; l < g->n; ++l)
        if (!grow(&g->stage_y[l], &g->stage_y_bytes[l], (size_t)M * g->h[l]->N * 2))
            return fail(PATCH_ERR_NOMEM, "staging allocation failed");

    // Token chunks: chunk c's inputs land while chunk c-1 computes and chunk
    // c-2's outputs go back (the two copy directions use separate engines).
    // Every chunk runs the kernel a device call with this M would run, and
    // chunks are whole multiples of its token tile, so each output element
    // comes from the same MMA sequence: the bits equal patch_group_linear's.
    const int rpath = resolve_path(g, path, M);
    const int64_t bn = (rpath == PATCH_PATH_GEMM_WIDE || rpath == PATCH_PATH_GEMM_WIDE_24) ? kGemm22BN
                       : rpath == PATCH_PATH_GEMM_PAIR ? kGemm2BN
                       : rpath == PATCH_PATH_GEMM_SINGLE ? kGemmBN
                                                         : M;
    int64_t chunk = M;
    if (M >= 4 * bn) chunk = ((M + 3) / 4 + bn - 1) / bn * bn;
    const int nchunks = (int)((M + chunk - 1) / chunk);
    while ((int)g->chunk_ev.size() < 2 * nchunks) {
        cudaEvent_t e = nullptr;
        PATCH_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        g->chunk_ev.push_back(e);
    }
    PATCH_CUDA(cudaStreamWaitEvent(g->h2d, g->last_done, 0));
    PATCH_CUDA(cudaStreamWaitEvent(s, g->last_done, 0));
    for (int c = 0; c < nchunks; ++c) {
        const int64_t m0 = c * chunk, rows = std::min<int64_t>(chunk, M - m0);
        cudaEvent_t x_ready = g->chunk_ev[2 * c], y_ready = g->chunk_ev[2 * c + 1];
        for (int i = 0; i < nslots; ++i)
            PATCH_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(g->stage_x[i]) + m0 * slotK[i] * 2,
                                       static_cast<const uint8_t*>(src[i]) + m0 * slotK[i] * 2,
                                       (size_t)rows * slotK[i] * 2, cudaMemcpyHostToDevice, g->h2d));
        PATCH_CUDA(cudaEventRecord(x_ready, g->h2d));
        PATCH_CUDA(cudaStreamWaitEvent(s, x_ready, 0));
        const void* xs[kMaxGroup];
        void* ys[kMaxGroup];
        for (int l = 0; l < g->n; ++l) {
            xs[l] = static_cast<const uint8_t*>(g->stage_x[slot[l]]) + m0 * g->h[l]->K * 2;
            ys[l] = static_cast<uint8_t*>(g->stage_y[l]) + m0 * g->h[l]->N * 2;
        }
        st = run_group(g, xs, rows, ys, rpath, s);
        if (st != PATCH_OK) return st;
        PATCH_CUDA(cudaEventRecord(y_ready, s));
        PATCH_CUDA(cudaStreamWaitEvent(g->d2h, y_ready, 0));
        for (int l = 0; l < g->n; ++l)
            PATCH_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(Y_host[l]) + m0 * g->h[l]->N * 2,
                                       static_cast<const uint8_t*>(g->stage_y[l]) + m0 * g->h[l]->N * 2,
                                       (size_t)rows * g->h[l]->N * 2, cudaMemcpyDeviceToHost, g->d2h));
    }
    PATCH_CUDA(cudaEventRecord(g->last_done, g->d2h));
    PATCH_CUDA(cudaStreamWaitEvent(s, g->last_done, 0));  // Y_host is complete once `stream` is
    return PATCH_OK;
}

patch_status patch_selftest_wait(void* stream) {
    int dev = 0;
    PATCH_CUDA(cudaGetDevice(&dev));
    patch_status st = check_device_is(dev);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = nullptr;
    if (cudaMalloc(&status, sizeof(int)) != cudaSuccess) return fail(PATCH_ERR_NOMEM, "status word");
    int host = 0;
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (e == cudaSuccess) e = launch_selftest_wait(status, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(status);
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    if (host == kStatusTimeout) return fail(PATCH_ERR_TIMEOUT, "self-test: the bounded wait gave up as designed");
    return PATCH_OK;
}

patch_status patch_unpack(patch_handle h, void* W_masked_bf16, void* stream) {
    if (!h || !W_masked_bf16) return fail(PATCH_ERR_ARG, "handle and output must be non-NULL");
    if (!aligned16(W_masked_bf16)) return fail(PATCH_ERR_ALIGN, "output must be 16-byte aligned");
    patch_status st = check_device_is(h->device);
    if (st != PATCH_OK) return st;
    unpack_kernel<<<h->plan.S * h->plan.KB, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        h->packed, h->slab_dev, h->meta_dev, h->plan.KB, h->plan.KC, h->K, static_cast<uint16_t*>(W_masked_bf16));
    PATCH_CUDA(cudaGetLastError());
    return PATCH_OK;
}

patch_status patch_info(patch_handle h, patch_info_t* info) {
    if (!h || !info) return fail(PATCH_ERR_ARG, "handle and info must be non-NULL");
    *info = h->info;
    return PATCH_OK;
}

patch_status patch_copy_packed(patch_handle h, void* packed_host, int64_t packed_cap, uint32_t* slab_host,
                               int64_t slab_cap, uint32_t* meta_host, int64_t meta_cap, uint32_t* gemm_host,
                               int64_t gemm_cap) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    const Plan& p = h->plan;
    if ((packed_host && packed_cap < p.bytes) || (slab_host && slab_cap < (int64_t)p.slab.size()) ||
        (meta_host && meta_cap < (int64_t)p.meta.size()) || (gemm_host && gemm_cap < (int64_t)p.gemm.size()))
        return fail(PATCH_ERR_ARG, "a destination buffer is too small");
    if (packed_host) PATCH_CUDA(cudaMemcpy(packed_host, h->packed, p.bytes, cudaMemcpyDeviceToHost));
    if (slab_host) memcpy(slab_host, p.slab.data(), sizeof(uint32_t) * p.slab.size());
    if (meta_host) memcpy(meta_host, p.meta.data(), sizeof(uint32_t) * p.meta.size());
    if (gemm_host) memcpy(gemm_host, p.gemm.data(), sizeof(uint32_t) * p.gemm.size());
    return PATCH_OK;
}

patch_status patch_check(patch_handle h, void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int word = 0;
    PATCH_CUDA(cudaStreamSynchronize(s));
    PATCH_CUDA(cudaMemcpy(&word, h->status_dev, sizeof(int), cudaMemcpyDeviceToHost));
    if (word != 0) {
        PATCH_CUDA(cudaDeviceSynchronize());
        PATCH_CUDA(cudaMemset(h->status_dev, 0, sizeof(int)));
        // an abandoned decode call may leave strip counters part-way: re-arm
        // those of every workspace of every group this handle belongs to
        std::vector<patch_group_s*> gs;
        {
            std::lock_guard<std::mutex> lk(h->groups_mu);
            gs = h->groups;
        }
        for (patch_group g : gs) {
            std::lock_guard<std::mutex> lk(g->mu);
            std::vector<DecodeWs*> all{&g->capture_ws};
            for (auto& kv : g->decode_ws) all.push_back(&kv.second);
            for (DecodeWs* w : all)
                for (int i = 0; i < g->n; ++i)
                    if (w->counters[i]) PATCH_CUDA(cudaMemset(w->counters[i], 0, sizeof(unsigned) * w->S[i]));
        }
        if (word == kStatusTimeout) return fail(PATCH_ERR_TIMEOUT, "a device-side wait ran past its limit");
        return fail(PATCH_ERR_CUDA, "device status word %d", word);
    }
    return PATCH_OK;
}

void patch_free(patch_handle h) { free_handle(h); }

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of patch_linear.
//
// The tensor-core kernels read their per-launch schedule (which output tiles
// each persistent CTA or CTA pair takes) from device memory that patch_linear
// allocates and caches per handle on the first call for each M. Callers that
// must not allocate device memory during the call (an allocator that is frozen
// after start-up, a memory pool owned by another framework, a host thread
// that may not touch the CUDA allocator) use patch_linear_noalloc instead: it
// writes the schedule into one fixed array that lives in this library's
// device image, so the call itself allocates nothing.
namespace {

constexpr int kNoAllocMaxSlots = 256;      // persistent CTAs or CTA pairs
constexpr int kNoAllocMaxUnits = 65536;    // output tiles of one call
constexpr int kNoAllocInts = (kNoAllocMaxSlots + 1) + kNoAllocMaxUnits;

// Schedule scratch shared by every call on a device: [0, slots] offsets, then
// the tile list. Host code must not pass this symbol to a kernel: its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) int g_noalloc_sched[kNoAllocInts];

std::mutex g_noalloc_mu;
std::map<int, int*> g_noalloc_addr;  // device -> device address of g_noalloc_sched

patch_status noalloc_scratch(int dev, int** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_addr.find(dev);
    if (it == g_noalloc_addr.end()) {
        int* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_sched);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the schedule scratch");
        it = g_noalloc_addr.emplace(dev, p).first;
    }
    *out = it->second;
    return PATCH_OK;
}

}  // namespace

extern "C" patch_status patch_linear_noalloc(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16,
                                             void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (M == 0) return PATCH_OK;
    patch_status s = check_xy(X_bf16, Y_bf16);
    if (s != PATCH_OK) return s;
    if (M > (int64_t)INT32_MAX / 2) return fail(PATCH_ERR_SHAPE, "M too large");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = check_device_is(h->device)) != PATCH_OK) return s;
    // Decode sizes: the CUDA-core kernel needs no schedule and no scratch.
    if (M <= 8) return run_simt(h, X_bf16, M, Y_bf16, st);
    const int path = resolve_path(h->self, PATCH_PATH_GEMM, M);
    const int kernel = choose_kernel(h->self, path, M);
    const int bn = kernel_bn(kernel);
    const int64_t mb = (M + bn - 1) / bn;
    const int64_t rows = kernel_rows(h->plan, kernel);
    const int slots = kernel_slots(h->dev, kernel);
    if (slots > kNoAllocMaxSlots)
        return fail(PATCH_ERR_UNSUPPORTED,
                    "patch_linear_noalloc holds schedules for at most %d persistent CTAs or CTA pairs "
                    "(this device runs %d); use patch_linear",
                    kNoAllocMaxSlots, slots);
    if (rows * mb > kNoAllocMaxUnits)
        return fail(PATCH_ERR_SHAPE,
                    "patch_linear_noalloc handles at most %d output tiles per call (this call needs %lld); "
                    "use patch_linear",
                    kNoAllocMaxUnits, (long long)(rows * mb));
    int* sched = nullptr;
    if ((s = noalloc_scratch(h->device, &sched)) != PATCH_OK) return s;
    std::vector<int> off, work;
    lpt_schedule(h->self, kernel, (int)mb, off, work);
    int* d_off = sched;
    int* d_work = sched + kNoAllocMaxSlots + 1;
    PATCH_CUDA(cudaMemcpyAsync(d_off, off.data(), sizeof(int) * off.size(), cudaMemcpyHostToDevice, st));
    PATCH_CUDA(cudaMemcpyAsync(d_work, work.data(), sizeof(int) * std::max<size_t>(work.size(), 1),
                               cudaMemcpyHostToDevice, st));
    const void* xs[1] = {X_bf16};
    void* ys[1] = {Y_bf16};
    return run_group(h->self, xs, M, ys, path, st, d_off, d_work, (int)off.size() - 1);
}
