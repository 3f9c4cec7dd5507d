// Host runtime behind the C ABI in patch_hybrid.h: argument checks, the slab
// table, the cost-balanced persistent schedule, tensor maps and launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include "kernels.cuh"
#include "patch_hybrid.h"

using namespace patch;

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

patch_status check_shape(int64_t N, int64_t K, int tile_rows, int tile_cols) {
    const bool shape_ok = (tile_rows == 128 || tile_rows == 64) && (tile_cols == 128 || tile_cols == 64);
    if (!shape_ok)
        return fail(PATCH_ERR_SHAPE, "tile shape %dx%d is not one of 128x128, 128x64, 64x128, 64x64", tile_rows,
                    tile_cols);
    if (N <= 0 || K <= 0) return fail(PATCH_ERR_SHAPE, "N and K must be positive");
    if (N % 128 || K % 64 || N % tile_rows || K % tile_cols)
        return fail(PATCH_ERR_SHAPE,
                    "need N %% 128 == 0, K %% 64 == 0 and both divisible by the tile (N=%lld K=%lld)",
                    (long long)N, (long long)K);
    if (N > (1 << 24) || K > (1 << 24) || N * K > ((int64_t)1 << 36)) return fail(PATCH_ERR_SHAPE, "weight too large");
    return PATCH_OK;
}

patch_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PATCH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define PATCH_CUDA(call)                                   \
    do {                                                   \
        cudaError_t e_ = (call);                           \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

patch_status check_device(int* dev_out, int* sms_out) {
    int dev = 0;
    PATCH_CUDA(cudaGetDevice(&dev));
    int major = 0, sms = 0;
    PATCH_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    PATCH_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    if (major != 10) return fail(PATCH_ERR_UNSUPPORTED, "device %d has compute capability %d.x, need 10.x", dev, major);
    *dev_out = dev;
    *sms_out = sms;
    return PATCH_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
std::mutex g_prep_mu;
std::map<int, bool> g_prepared;  // per device: kernel attributes set

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

patch_status prepare_device(int dev) {
    std::lock_guard<std::mutex> lk(g_prep_mu);
    if (g_prepared[dev]) return PATCH_OK;
    PATCH_CUDA(gemm_prepare());
    g_prepared[dev] = true;
    return PATCH_OK;
}

struct WorkList {
    int grid = 0;
    int* off = nullptr;   // device, grid + 1
    int* work = nullptr;  // device, units
};

}  // namespace

struct patch_handle_s {
    int device = 0;
    int sms = 0;
    int64_t N = 0, K = 0;
    int R = 0, C = 0, S = 0, KB = 0;
    uint8_t* packed = nullptr;
    int64_t packed_bytes = 0;
    uint32_t* table_dev = nullptr;
    std::vector<uint32_t> table;
    std::vector<double> strip_cost;
    int* status_dev = nullptr;
    patch_info_t info{};
    std::mutex mu;
    std::map<std::pair<int, int>, WorkList> work;  // (bn, m_blocks) -> schedule
    void* stage_x = nullptr;
    size_t stage_x_bytes = 0;
    void* stage_y = nullptr;
    size_t stage_y_bytes = 0;
};

namespace {

void free_handle(patch_handle h) {
    if (!h) return;
    cudaDeviceSynchronize();
    cudaFree(h->packed);
    cudaFree(h->table_dev);
    cudaFree(h->status_dev);
    for (auto& kv : h->work) {
        cudaFree(kv.second.off);
        cudaFree(kv.second.work);
    }
    cudaFree(h->stage_x);
    cudaFree(h->stage_y);
    delete h;
}

// Slab table: a slab (128 rows x 64 columns) is stored compressed only when
// every mask tile it overlaps is flagged 2:4; the first compressed slab of a
// 128-column chunk carries that chunk's metadata block.
int64_t build_table(patch_handle h, const uint8_t* flags) {
    const int64_t tiles_k = h->K / h->C;
    h->table.assign((size_t)h->S * h->KB, 0u);
    h->strip_cost.assign(h->S, 0.0);
    int64_t off = 0, sparse_slabs = 0;
    for (int s = 0; s < h->S; ++s) {
        int meta_chunk = -1;
        for (int b = 0; b < h->KB; ++b) {
            bool sp = true;
            for (int r0 = s * kStrip; r0 < (s + 1) * kStrip; r0 += h->R)
                sp = sp && flags[(int64_t)(r0 / h->R) * tiles_k + ((int64_t)b * kSlabK) / h->C] != 0;
            bool meta = false;
            if (sp && meta_chunk != b / 2) {
                meta = true;
                meta_chunk = b / 2;
            }
            h->table[(size_t)s * h->KB + b] =
                (uint32_t)((off / 16) << 2) | (meta ? kSlabHasMeta : 0u) | (sp ? kSlabSparse : 0u);
            off += sp ? kSparseValBytes + (meta ? kMetaBytes : 0) : kDenseSlabBytes;
            sparse_slabs += sp;
            h->strip_cost[s] += sp ? 0.5 : 1.0;
        }
    }
    h->info.slabs_total = (int64_t)h->S * h->KB;
    h->info.slabs_sparse = sparse_slabs;
    return off;
}

// Greedy longest-processing-time assignment of output tiles (strip, token
// block) to persistent CTAs. A tile's cost is its slab work (dense 1, sparse
// 1/2, the ratio of tensor-core time) plus a fixed epilogue share.
patch_status get_worklist(patch_handle h, int bn, int mb, WorkList** out) {
    std::lock_guard<std::mutex> lk(h->mu);
    auto key = std::make_pair(bn, mb);
    auto it = h->work.find(key);
    if (it != h->work.end()) {
        *out = &it->second;
        return PATCH_OK;
    }
    const int units = h->S * mb;
    const int grid = std::max(1, std::min(h->sms, units));
    std::vector<int> order(units);
    for (int u = 0; u < units; ++u) order[u] = u;
    const double epi = 1.0;
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
        return h->strip_cost[x / mb] > h->strip_cost[y / mb];
    });
    using Item = std::pair<double, int>;  // (load, cta)
    std::priority_queue<Item, std::vector<Item>, std::greater<Item>> pq;
    for (int c = 0; c < grid; ++c) pq.push({0.0, c});
    std::vector<std::vector<int>> lists(grid);
    for (int u : order) {
        Item top = pq.top();
        pq.pop();
        lists[top.second].push_back(u);
        top.first += h->strip_cost[u / mb] + epi;
        pq.push(top);
    }
    std::vector<int> off(grid + 1, 0), work;
    work.reserve(units);
    for (int c = 0; c < grid; ++c) {
        off[c] = (int)work.size();
        work.insert(work.end(), lists[c].begin(), lists[c].end());
    }
    off[grid] = (int)work.size();
    WorkList wl;
    wl.grid = grid;
    if (cudaMalloc(&wl.off, sizeof(int) * (grid + 1)) != cudaSuccess ||
        cudaMalloc(&wl.work, sizeof(int) * std::max(units, 1)) != cudaSuccess) {
        cudaFree(wl.off);
        return fail(PATCH_ERR_NOMEM, "schedule allocation failed");
    }
    PATCH_CUDA(cudaMemcpy(wl.off, off.data(), sizeof(int) * (grid + 1), cudaMemcpyHostToDevice));
    PATCH_CUDA(cudaMemcpy(wl.work, work.data(), sizeof(int) * units, cudaMemcpyHostToDevice));
    auto res = h->work.emplace(key, wl);
    *out = &res.first->second;
    return PATCH_OK;
}

patch_status make_x_map(CUtensorMap* map, const void* X, int64_t M, int64_t K, int bn) {
    patch_status st = get_encode();
    if (st != PATCH_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kSlabK, (cuuint32_t)bn};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PATCH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PATCH_OK;
}

patch_status check_handle_device(patch_handle h) {
    int dev = -1;
    PATCH_CUDA(cudaGetDevice(&dev));
    if (dev != h->device) return fail(PATCH_ERR_ARG, "handle lives on device %d, current device is %d", h->device, dev);
    return PATCH_OK;
}

patch_status run_linear(patch_handle h, const void* X, int64_t M, void* Y, int path, cudaStream_t st) {
    if (path == PATCH_PATH_AUTO) path = (M <= 8) ? PATCH_PATH_GEMV : PATCH_PATH_GEMM;
    if (path == PATCH_PATH_GEMV) {
        if (M > 16) return fail(PATCH_ERR_SHAPE, "the decode kernel takes M <= 16 (got %lld)", (long long)M);
        GemvArgs a;
        a.packed = h->packed;
        a.table = h->table_dev;
        a.X = static_cast<const __nv_bfloat16*>(X);
        a.Y = static_cast<__nv_bfloat16*>(Y);
        a.M = (int)M;
        a.N = (int)h->N;
        a.K = (int)h->K;
        a.KB = h->KB;
        cudaError_t e = launch_gemv(a, st);
        if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
        return PATCH_OK;
    }
    if (path != PATCH_PATH_GEMM) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    if (M > (int64_t)INT32_MAX / 2) return fail(PATCH_ERR_SHAPE, "M too large");
    const int bn = gemm_bn_for((int)M);
    const int mb = (int)((M + bn - 1) / bn);
    WorkList* wl = nullptr;
    patch_status s = get_worklist(h, bn, mb, &wl);
    if (s != PATCH_OK) return s;
    CUtensorMap map;
    s = make_x_map(&map, X, M, h->K, bn);
    if (s != PATCH_OK) return s;
    GemmArgs a;
    a.packed = h->packed;
    a.table = h->table_dev;
    a.work_off = wl->off;
    a.work = wl->work;
    a.M = (int)M;
    a.N = (int)h->N;
    a.KB = h->KB;
    a.MB = mb;
    a.Y = static_cast<__nv_bfloat16*>(Y);
    a.status = h->status_dev;
    cudaError_t e = launch_gemm(map, a, wl->grid, bn, st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel launch");
    return PATCH_OK;
}

}  // namespace

extern "C" {

const char* patch_last_error(void) { return g_err.c_str(); }

int patch_version(void) { return 1; }

patch_status patch_pack(const void* W_bf16, int64_t N, int64_t K, const uint8_t* mask_bits, int bitorder,
                        const uint8_t* tile_flags, int tile_rows, int tile_cols, void* stream,
                        patch_handle* out) {
    g_err.clear();
    if (!out) return fail(PATCH_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (!W_bf16 || !mask_bits || !tile_flags) return fail(PATCH_ERR_ARG, "W, mask_bits and tile_flags must be non-NULL");
    if (bitorder != 0 && bitorder != 1) return fail(PATCH_ERR_ARG, "bitorder must be 0 or 1");
    {
        patch_status sst = check_shape(N, K, tile_rows, tile_cols);
        if (sst != PATCH_OK) return sst;
    }
    if (!aligned16(W_bf16)) return fail(PATCH_ERR_ALIGN, "W must be 16-byte aligned");
    int dev = 0, sms = 0;
    patch_status st = check_device(&dev, &sms);
    if (st != PATCH_OK) return st;
    st = prepare_device(dev);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    patch_handle h = new (std::nothrow) patch_handle_s();
    if (!h) return fail(PATCH_ERR_NOMEM, "host allocation failed");
    h->device = dev;
    h->sms = sms;
    h->N = N;
    h->K = K;
    h->R = tile_rows;
    h->C = tile_cols;
    h->S = (int)(N / kStrip);
    h->KB = (int)(K / kSlabK);
    const int64_t ntiles = (N / tile_rows) * (K / tile_cols);
    int64_t tiles_sparse = 0;
    for (int64_t i = 0; i < ntiles; ++i) {
        if (tile_flags[i] > 1) {
            free_handle(h);
            return fail(PATCH_ERR_ARG, "tile flag %lld is %d, must be 0 or 1", (long long)i, (int)tile_flags[i]);
        }
        tiles_sparse += tile_flags[i];
    }
    h->packed_bytes = build_table(h, tile_flags);
    if (h->packed_bytes / 16 >= ((int64_t)1 << 30)) {
        free_handle(h);
        return fail(PATCH_ERR_SHAPE, "packed weight exceeds the 16 GiB slab-table range");
    }

    uint8_t* flags_dev = nullptr;
    unsigned long long* counters = nullptr;
    auto cleanup = [&](patch_status code) {
        cudaFree(flags_dev);
        cudaFree(counters);
        if (code != PATCH_OK) free_handle(h);
        return code;
    };
    if (cudaMalloc(&h->packed, std::max<int64_t>(h->packed_bytes, 16)) != cudaSuccess ||
        cudaMalloc(&h->table_dev, sizeof(uint32_t) * h->table.size()) != cudaSuccess ||
        cudaMalloc(&h->status_dev, sizeof(int)) != cudaSuccess || cudaMalloc(&flags_dev, ntiles) != cudaSuccess ||
        cudaMalloc(&counters, 3 * sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        return cleanup(fail(PATCH_ERR_NOMEM, "device allocation of %lld packed bytes failed", (long long)h->packed_bytes));
    }
    cudaError_t e;
    if ((e = cudaMemcpyAsync(h->table_dev, h->table.data(), sizeof(uint32_t) * h->table.size(),
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
    a.table = h->table_dev;
    a.out = h->packed;
    a.K = K;
    a.R = tile_rows;
    a.C = tile_cols;
    a.KB = h->KB;
    a.counters = counters;
    pack_kernel<<<h->S * h->KB, 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return cleanup(cuda_fail(e, "pack kernel launch"));
    unsigned long long cnt[3] = {0, 0, 0};
    if ((e = cudaMemcpyAsync(cnt, counters, sizeof(cnt), cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
        return cleanup(cuda_fail(e, "pack kernel"));
    if (cnt[0] != 0)
        return cleanup(fail(PATCH_ERR_MASK, "%llu groups inside 2:4 tiles do not keep exactly two of four", cnt[0]));
    h->info.N = N;
    h->info.K = K;
    h->info.tile_rows = tile_rows;
    h->info.tile_cols = tile_cols;
    h->info.tiles_total = ntiles;
    h->info.tiles_sparse = tiles_sparse;
    h->info.packed_bytes = h->packed_bytes;
    h->info.pruned = (int64_t)cnt[2];
    h->info.stray_zeros = (int64_t)cnt[1];
    h->info.sparsity = (double)cnt[2] / (double)(N * K);
    *out = h;
    return cleanup(PATCH_OK);
}

patch_status patch_linear_path(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16, int path,
                               void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (M == 0) return PATCH_OK;
    if (!X_bf16 || !Y_bf16) return fail(PATCH_ERR_ARG, "X and Y must be non-NULL");
    if (!aligned16(X_bf16) || !aligned16(Y_bf16)) return fail(PATCH_ERR_ALIGN, "X and Y must be 16-byte aligned");
    if (path < PATCH_PATH_AUTO || path > PATCH_PATH_GEMV) return fail(PATCH_ERR_ARG, "unknown path %d", path);
    patch_status st = check_handle_device(h);
    if (st != PATCH_OK) return st;
    return run_linear(h, X_bf16, M, Y_bf16, path, static_cast<cudaStream_t>(stream));
}

patch_status patch_linear(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16, void* stream) {
    return patch_linear_path(h, X_bf16, M, Y_bf16, PATCH_PATH_AUTO, stream);
}

patch_status patch_linear_host(patch_handle h, const void* X_host, int64_t M, void* Y_host, void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (M < 0) return fail(PATCH_ERR_ARG, "M must be >= 0");
    if (M == 0) return PATCH_OK;
    if (!X_host || !Y_host) return fail(PATCH_ERR_ARG, "X and Y must be non-NULL");
    patch_status st = check_handle_device(h);
    if (st != PATCH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t xb = (size_t)M * h->K * 2, yb = (size_t)M * h->N * 2;
    if (xb > h->stage_x_bytes) {
        cudaFree(h->stage_x);
        h->stage_x = nullptr;
        h->stage_x_bytes = 0;
        if (cudaMalloc(&h->stage_x, xb) != cudaSuccess) return fail(PATCH_ERR_NOMEM, "staging allocation failed");
        h->stage_x_bytes = xb;
    }
    if (yb > h->stage_y_bytes) {
        cudaFree(h->stage_y);
        h->stage_y = nullptr;
        h->stage_y_bytes = 0;
        if (cudaMalloc(&h->stage_y, yb) != cudaSuccess) return fail(PATCH_ERR_NOMEM, "staging allocation failed");
        h->stage_y_bytes = yb;
    }
    PATCH_CUDA(cudaMemcpyAsync(h->stage_x, X_host, xb, cudaMemcpyHostToDevice, s));
    st = run_linear(h, h->stage_x, M, h->stage_y, PATCH_PATH_AUTO, s);
    if (st != PATCH_OK) return st;
    PATCH_CUDA(cudaMemcpyAsync(Y_host, h->stage_y, yb, cudaMemcpyDeviceToHost, s));
    PATCH_CUDA(cudaStreamSynchronize(s));
    return PATCH_OK;
}

patch_status patch_unpack(patch_handle h, void* W_masked_bf16, void* stream) {
    if (!h || !W_masked_bf16) return fail(PATCH_ERR_ARG, "handle and output must be non-NULL");
    if (!aligned16(W_masked_bf16)) return fail(PATCH_ERR_ALIGN, "output must be 16-byte aligned");
    patch_status st = check_handle_device(h);
    if (st != PATCH_OK) return st;
    unpack_kernel<<<h->S * h->KB, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        h->packed, h->table_dev, h->KB, h->K, static_cast<uint16_t*>(W_masked_bf16));
    PATCH_CUDA(cudaGetLastError());
    return PATCH_OK;
}

patch_status patch_info(patch_handle h, patch_info_t* info) {
    if (!h || !info) return fail(PATCH_ERR_ARG, "handle and info must be non-NULL");
    *info = h->info;
    return PATCH_OK;
}

patch_status patch_copy_packed(patch_handle h, void* packed_host, int64_t packed_cap, uint32_t* table_host,
                               int64_t table_cap) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    if (packed_host) {
        if (packed_cap < h->packed_bytes) return fail(PATCH_ERR_ARG, "packed buffer too small");
        PATCH_CUDA(cudaMemcpy(packed_host, h->packed, h->packed_bytes, cudaMemcpyDeviceToHost));
    }
    if (table_host) {
        if (table_cap < (int64_t)h->table.size()) return fail(PATCH_ERR_ARG, "table buffer too small");
        memcpy(table_host, h->table.data(), sizeof(uint32_t) * h->table.size());
    }
    return PATCH_OK;
}

patch_status patch_check(patch_handle h, void* stream) {
    if (!h) return fail(PATCH_ERR_ARG, "handle is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int word = 0;
    PATCH_CUDA(cudaStreamSynchronize(s));
    PATCH_CUDA(cudaMemcpy(&word, h->status_dev, sizeof(int), cudaMemcpyDeviceToHost));
    if (word != 0) {
        PATCH_CUDA(cudaMemset(h->status_dev, 0, sizeof(int)));
        if (word == kStatusTimeout) return fail(PATCH_ERR_TIMEOUT, "a device-side wait ran past its limit");
        return fail(PATCH_ERR_CUDA, "device status word %d", word);
    }
    return PATCH_OK;
}

void patch_free(patch_handle h) { free_handle(h); }

patch_status patch_plan(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows, int tile_cols,
                        uint32_t* table_host, int64_t* packed_bytes) {
    g_err.clear();
    if (!tile_flags) return fail(PATCH_ERR_ARG, "tile_flags is NULL");
    patch_status st = check_shape(N, K, tile_rows, tile_cols);
    if (st != PATCH_OK) return st;
    const int64_t ntiles = (N / tile_rows) * (K / tile_cols);
    for (int64_t i = 0; i < ntiles; ++i)
        if (tile_flags[i] > 1) return fail(PATCH_ERR_ARG, "tile flag %lld is %d, must be 0 or 1", (long long)i, (int)tile_flags[i]);
    patch_handle_s tmp;
    tmp.N = N;
    tmp.K = K;
    tmp.R = tile_rows;
    tmp.C = tile_cols;
    tmp.S = (int)(N / kStrip);
    tmp.KB = (int)(K / kSlabK);
    const int64_t bytes = build_table(&tmp, tile_flags);
    if (table_host) memcpy(table_host, tmp.table.data(), sizeof(uint32_t) * tmp.table.size());
    if (packed_bytes) *packed_bytes = bytes;
    return PATCH_OK;
}

}  // extern "C"
