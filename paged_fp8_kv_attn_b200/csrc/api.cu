// api.cu -- the extern "C" entry points declared in include/pagedkv.h:
// host-side argument validation, TMA descriptor encoding, workspace layout
// and kernel launches.  No call allocates, frees or synchronises.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "internal.h"
#include "pagedkv.h"

namespace {

thread_local std::string g_last_error;

pkv_status fail(pkv_status code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

pkv_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool supported_head_dim(int32_t d) { return d == 64 || d == 128; }
bool supported_page_size(int32_t p) { return p == 16 || p == 32 || p == 64 || p == 128; }

// ---------------------------------------------------------------------------
// per-device launch limits (SM count, resident attention CTAs per SM)
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int occupancy[2][2][2][2] = {};   // [fp8][d128][gp16][two KV heads per item]
    // resident clusters of each size (index = cluster size; -1 = not queried)
    int clusters[2][2][2][2][pkv::kMaxCluster + 1];
};
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

pkv_status device_info(const DeviceInfo** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& info = g_dev[dev];
    if (!info.ready) {
        e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        e = pkv::step_kernels_set_carveout();
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        for (int f = 0; f < 2; ++f)
            for (int d = 0; d < 2; ++d)
                for (int gp = 0; gp < 2; ++gp)
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const bool fp8 = f == 1;
                        const int hd = d ? 128 : 64, gpad = gp ? 16 : 8, kvh = h2 ? 2 : 1;
                        if (pkv::attn_partial_smem_bytes(fp8, hd, gpad, kvh) == 0) continue;
                        e = pkv::attn_set_smem_attr(fp8, hd, gpad, kvh);
                        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
                        int blocks = 0;
                        e = pkv::attn_occupancy(fp8, hd, gpad, kvh, &blocks);
                        if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
                        info.occupancy[f][d][gp][h2] = blocks < 1 ? 1 : blocks;
                        for (int c = 0; c <= pkv::kMaxCluster; ++c) info.clusters[f][d][gp][h2][c] = -1;
                    }
        info.ready = true;
    }
    *out = &info;
    return PKV_OK;
}

int group_pad_of(int group) { return group <= 8 ? 8 : 16; }

// Clusters of `size` CTAs of this attention variant that fit on the device at
// once (queried once per device, variant and size).
pkv_status max_clusters(bool fp8, int head_dim, int group, int kv_per_item, int size, int* out) {
    const DeviceInfo* cinfo = nullptr;
    pkv_status st = device_info(&cinfo);
    if (st != PKV_OK) return st;
    DeviceInfo& info = const_cast<DeviceInfo&>(*cinfo);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    int& slot = info.clusters[fp8 ? 1 : 0][head_dim == 128][group > 8][kv_per_item == 2][size];
    if (slot < 0) {
        int n = 0;
        cudaError_t e = pkv::attn_max_clusters(fp8, head_dim, group_pad_of(group), kv_per_item,
                                               size, &n);
        if (e != cudaSuccess) {
            cudaGetLastError();   // a refused shape is an answer, not a sticky error
            n = 0;
        }
        slot = n;
    }
    *out = slot;
    return PKV_OK;
}

// Cluster mode for `items` work items: cluster size C and K clusters, each
// owning ceil(items / K) or fewer whole items.  With `forced` > 0 the size is
// given; otherwise the size maximising C * items / (items per cluster) -- the
// CTAs kept busy, discounted by the imbalance of whole items per cluster --
// over 2..kMaxCluster.  Among sizes that tie, the largest portable one (at
// most 8) wins: more CTAs share each cluster's items, which evens out
// requests of unequal length.  Returns C = 0 when no cluster shape fits.
pkv_status choose_clusters(bool fp8, int head_dim, int group, int kv_per_item, int64_t items,
                           int forced, int* size, int* count) {
    *size = 0;
    *count = 0;
    double best = 0.0;
    const int c_lo = forced > 0 ? forced : 2;
    const int c_hi = forced > 0 ? forced : pkv::kMaxCluster;
    for (int c = c_lo; c <= c_hi; ++c) {
        int kmax = 0;
        pkv_status st = max_clusters(fp8, head_dim, group, kv_per_item, c, &kmax);
        if (st != PKV_OK) return st;
        if (kmax <= 0) continue;
        const int64_t k = std::min<int64_t>(items, kmax);
        const int64_t per = (items + k - 1) / k;            // items of the fullest cluster
        const double score = static_cast<double>(c) * static_cast<double>(items) / per;
        if (score > best || (score == best && c <= 8)) {
            best = score;
            *size = c;
            *count = static_cast<int>((items + per - 1) / per);
        }
    }
    return PKV_OK;
}

pkv_status default_ctas(bool fp8, int head_dim, int group, int kv_per_item, int* ctas) {
    const DeviceInfo* info = nullptr;
    pkv_status st = device_info(&info);
    if (st != PKV_OK) return st;
    *ctas = info->sms * info->occupancy[fp8 ? 1 : 0][head_dim == 128][group > 8][kv_per_item == 2];
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors for the K / V pools viewed as 2-D [rows][head_dim]
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

pkv_status get_encoder(EncodeTiledFn* fn) {
    static std::once_flag once;
    static EncodeTiledFn cached = nullptr;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            cached = reinterpret_cast<EncodeTiledFn>(p);
    });
    if (cached == nullptr)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
    *fn = cached;
    return PKV_OK;
}

pkv_status encode_pool_map(CUtensorMap* map, const void* pool, bool fp8, int head_dim,
                           int64_t rows, int box_rows) {
    EncodeTiledFn encode = nullptr;
    pkv_status st = get_encoder(&encode);
    if (st != PKV_OK) return st;
    const int esize = fp8 ? 1 : 2;
    const int box_inner = fp8 ? head_dim : 64;  // elements; 64 or 128 bytes
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * esize};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw =
        (box_inner * esize == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        2, const_cast<void*>(pool), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PKV_OK;
}

// Generic 2-D map: `rows` rows of `inner` elements, rows `row_bytes` apart.
pkv_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                     uint64_t inner, uint64_t rows, uint64_t row_bytes, uint32_t box_inner,
                     uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn encode = nullptr;
    pkv_status st = get_encoder(&encode);
    if (st != PKV_OK) return st;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PKV_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

pkv_status check_common_kv(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                           int32_t page_size, int32_t num_pages, int32_t max_pages) {
    if (batch < 0) return fail(PKV_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", batch);
    if (num_kv_heads < 1) return fail(PKV_ERR_INVALID_ARG, "num_kv_heads must be >= 1");
    if (!supported_head_dim(head_dim))
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
    if (!supported_page_size(page_size))
        return fail(PKV_ERR_UNSUPPORTED, "page_size %d not supported (16, 32, 64, 128)", page_size);
    if (num_pages < 1) return fail(PKV_ERR_INVALID_ARG, "num_pages must be >= 1");
    if (max_pages < 1) return fail(PKV_ERR_INVALID_ARG, "max_pages must be >= 1");
    const int64_t rows = static_cast<int64_t>(num_pages) * num_kv_heads * page_size;
    if (rows >= (int64_t(1) << 31))
        return fail(PKV_ERR_UNSUPPORTED, "num_pages * num_kv_heads * page_size must be < 2^31");
    return PKV_OK;
}

// The work split of one attention call (see paged_decode_attn_plan).
struct AttnPlan {
    int kv_per_item;      // KV heads per work item the kernel uses
    int ws_kv_per_item;   // the one the workspace is sized for
    int grid;             // split-K grid (also sizes the workspace)
    int cluster;          // 0: split-K + merge; C > 0: clusters of C CTAs
    int nclusters;
};

pkv_status plan_attention(bool fp8, int32_t batch, int32_t num_kv_heads, int32_t group,
                          int32_t head_dim, int32_t max_pages, int32_t page_size,
                          int32_t num_ctas, AttnPlan* plan, bool allow_cluster = true) {
    pkv_status st = PKV_OK;
    int kv_per_item = pkv::kv_heads_per_item(fp8, num_kv_heads, group);
    plan->ws_kv_per_item = kv_per_item;
    int grid = num_ctas > 0 ? num_ctas : 0;
    if (grid == 0) {
        // one wave of resident CTAs, but no more than leaves each CTA about
        // eight 64-token chunks of the largest batch the page table allows
        // (small batches gain from fewer, longer segments and a lighter merge)
        st = default_ctas(fp8, head_dim, group, kv_per_item, &grid);
        if (st != PKV_OK) return st;
        const DeviceInfo* info = nullptr;
        st = device_info(&info);
        if (st != PKV_OK) return st;
        const int64_t chunks_per_seq =
            (static_cast<int64_t>(max_pages) * page_size + pkv::kChunkTokens - 1) / pkv::kChunkTokens;
        const int64_t max_units =
            static_cast<int64_t>(batch) * (num_kv_heads / kv_per_item) * chunks_per_seq;
        const int64_t cap = std::max<int64_t>(info->sms, (max_units + 7) / 8);
        if (cap < grid) grid = static_cast<int>(cap);
    } else {
        const DeviceInfo* info = nullptr;
        st = device_info(&info);  // sets the shared-memory attribute
        if (st != PKV_OK) return st;
    }
    plan->grid = grid;
    // Cluster mode (no merge kernel): the library's choice (num_ctas == 0)
    // when the batch has no more items than one wave of CTAs (measured on
    // B200: faster than split-K plus merge at every such size of the
    // concurrency sweep; larger batches, which can be ragged, keep the
    // balanced split-K partition), or requested with num_ctas = -C.  With at
    // most a quarter as many two-head items as SMs (up to 9 requests at 8 KV
    // heads), the library's choice takes one KV head per item, which doubles
    // the items and the CTAs that share them (measured on B200 at 8,192
    // tokens: 13% faster at 4 requests, unchanged at 1 and 8, 4-5% slower at
    // 16 and 32; cluster mode needs the workspace for its status word only,
    // so the workspace size does not depend on this).
    int64_t items = static_cast<int64_t>(batch) * (num_kv_heads / kv_per_item);
    int cluster = 0, nclusters = 0;
    if (allow_cluster && (num_ctas < 0 || (num_ctas == 0 && items <= grid))) {
        if (num_ctas == 0 && kv_per_item == 2) {
            const DeviceInfo* info = nullptr;
            st = device_info(&info);
            if (st != PKV_OK) return st;
            if (items * 4 <= info->sms) {
                kv_per_item = 1;
                items *= 2;
            }
        }
        st = choose_clusters(fp8, head_dim, group, kv_per_item, items,
                             num_ctas < 0 ? -num_ctas : 0, &cluster, &nclusters);
        if (st != PKV_OK) return st;
        if (cluster == 0 && num_ctas < 0)
            return fail(PKV_ERR_UNSUPPORTED, "clusters of %d CTAs do not fit on this device",
                        -num_ctas);
    }
    plan->kv_per_item = kv_per_item;
    plan->cluster = cluster;
    plan->nclusters = nclusters;
    return PKV_OK;
}

pkv_status attn_impl(bool fp8, const uint16_t* q, const void* k_cache, const void* v_cache,
                     float k_scale, float v_scale, const int32_t* page_table, int32_t max_pages,
                     const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                     int32_t num_kv_heads, int32_t head_dim, int32_t page_size, int32_t num_pages,
                     float sm_scale, const uint8_t* abort, uint16_t* out, float* lse,
                     void* workspace, size_t workspace_bytes, int32_t num_ctas, void* stream) {
    pkv_status st = check_common_kv(batch, num_kv_heads, head_dim, page_size, num_pages, max_pages);
    if (st != PKV_OK) return st;
    if (num_q_heads < 1 || num_q_heads % num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of "
                    "num_kv_heads (%d)", num_q_heads, num_kv_heads);
    const int group = num_q_heads / num_kv_heads;
    if (group > 16) return fail(PKV_ERR_UNSUPPORTED, "GQA group %d > 16 not supported", group);
    if (!(std::isfinite(sm_scale)))
        return fail(PKV_ERR_INVALID_ARG, "sm_scale must be finite");
    if (fp8 && (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
                !std::isfinite(v_scale)))
        return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and > 0");
    if (num_ctas < -pkv::kMaxCluster)
        return fail(PKV_ERR_INVALID_ARG, "num_ctas must be >= %d (got %d)", -pkv::kMaxCluster,
                    num_ctas);
    if (batch == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out || !lse)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 4) ||
        !aligned(lse, 4) || !aligned(page_table, 4) || !aligned(seq_lens, 4))
        return fail(PKV_ERR_INVALID_ARG, "misaligned pointer (q and caches need 16 bytes)");
    if (!workspace || !aligned(workspace, 256))
        return fail(PKV_ERR_WORKSPACE, "workspace must be non-null and 256-byte aligned");

    AttnPlan plan;
    st = plan_attention(fp8, batch, num_kv_heads, group, head_dim, max_pages, page_size, num_ctas,
                        &plan);
    if (st != PKV_OK) return st;
    const int kv_per_item = plan.kv_per_item;
    const int grid = plan.grid;
    const int cluster = plan.cluster, nclusters = plan.nclusters;
    const pkv::WorkspaceLayout wl =
        pkv::workspace_layout(batch, group, num_kv_heads, plan.ws_kv_per_item, head_dim, grid);
    if (workspace_bytes < wl.total)
        return fail(PKV_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes,
                    wl.total);

    // rows of one TMA box: a 64-token chunk of a page (a whole page when
    // smaller); with two KV heads per item and 64-token pages, both heads' rows
    // of the page at once (they are adjacent in the pool)
    const int box_rows = (kv_per_item == 2 && page_size == pkv::kChunkTokens)
                             ? 2 * pkv::kChunkTokens
                             : (page_size < pkv::kChunkTokens ? page_size : pkv::kChunkTokens);
    const int64_t rows = static_cast<int64_t>(num_pages) * num_kv_heads * page_size;
    CUtensorMap tk, tv;
    st = encode_pool_map(&tk, k_cache, fp8, head_dim, rows, box_rows);
    if (st != PKV_OK) return st;
    st = encode_pool_map(&tv, v_cache, fp8, head_dim, rows, box_rows);
    if (st != PKV_OK) return st;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    pkv::AttnArgs a{};
    a.q = q;
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.abort = abort;
    a.out = out;
    a.lse = lse;
    a.ws_status = reinterpret_cast<uint32_t*>(ws);
    a.ws_ml = reinterpret_cast<float*>(ws + wl.ml_off);
    a.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
    a.batch = batch;
    a.max_pages = max_pages;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.kv_per_item = kv_per_item;
    a.items_per_req = num_kv_heads / kv_per_item;
    a.group = group;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.num_ctas = cluster > 0 ? cluster * nclusters : grid;
    a.box_rows = box_rows;
    a.cluster_size = cluster;
    a.num_clusters = nclusters;
    a.qk_scale = sm_scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
    a.v_scale = fp8 ? v_scale : 1.f;

    cudaError_t e = pkv::launch_attn_partial(fp8, head_dim, group_pad_of(group), kv_per_item,
                                             a.num_ctas, as_stream(stream), tk, tv, a);
    if (e != cudaSuccess) return cuda_fail(e, "attention partial launch");
    if (cluster == 0) {
        e = pkv::launch_attn_merge(head_dim, as_stream(stream), a);
        if (e != cudaSuccess) return cuda_fail(e, "attention merge launch");
    }
    return PKV_OK;
}

// Shared-prefix mode: the split-K workspace, then the prefix records and the
// plan arrays.
struct PrefixLayout {
    size_t pml_off, po_off, link_off, leader_off, refkey_off, ref_off, share_off, pshare_off,
        cbeg_off, tiles_off, ntiles_off, total;
};

bool prefix_supported(int32_t num_kv_heads, int32_t group, int32_t head_dim) {
    return head_dim == 128 && pkv::kv_heads_per_item(true, num_kv_heads, group) == 2;
}

PrefixLayout prefix_layout(size_t base, int32_t batch, int32_t num_kv_heads, int32_t group) {
    PrefixLayout l{};
    const size_t items = static_cast<size_t>(batch) * (num_kv_heads / 2);
    const size_t heads = 2 * static_cast<size_t>(group);
    const size_t B = static_cast<size_t>(batch);
    l.pml_off = round_up(base, 256);
    l.po_off = round_up(l.pml_off + items * heads * 4 * 4, 256);
    l.link_off = round_up(l.po_off + items * heads * 128 * 4, 256);
    l.leader_off = round_up(l.link_off + B * 4, 256);
    l.refkey_off = round_up(l.leader_off + B * 4, 256);
    l.ref_off = round_up(l.refkey_off + B * 8, 256);
    l.share_off = round_up(l.ref_off + B * 4, 256);
    l.pshare_off = round_up(l.share_off + B * 4, 256);
    l.cbeg_off = round_up(l.pshare_off + B * 4, 256);
    l.tiles_off = round_up(l.cbeg_off + B * 4, 256);
    l.ntiles_off = round_up(l.tiles_off + (B / 2 + 1) * 4 * 4, 256);
    l.total = round_up(l.ntiles_off + 4, 256);
    return l;
}

pkv_status prefix_impl(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                       float k_scale, float v_scale, const int32_t* page_table, int32_t max_pages,
                       const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                       int32_t num_pages, float sm_scale, const uint8_t* abort, uint16_t* out,
                       float* lse, void* workspace, size_t workspace_bytes, int32_t num_ctas,
                       int32_t* chunk_begin_out, void* stream) {
    pkv_status st = check_common_kv(batch, num_kv_heads, head_dim, page_size, num_pages, max_pages);
    if (st != PKV_OK) return st;
    if (num_q_heads < 1 || num_q_heads % num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of "
                    "num_kv_heads (%d)", num_q_heads, num_kv_heads);
    const int group = num_q_heads / num_kv_heads;
    if (num_ctas < 0)
        return fail(PKV_ERR_INVALID_ARG, "num_ctas must be >= 0 in shared-prefix mode (got %d)",
                    num_ctas);
    if (!prefix_supported(num_kv_heads, group, head_dim)) {
        // no shared-prefix tile for this shape: the plain call, no chunk shared
        st = attn_impl(true, q, k_cache, v_cache, k_scale, v_scale, page_table, max_pages,
                       seq_lens, batch, num_q_heads, num_kv_heads, head_dim, page_size, num_pages,
                       sm_scale, abort, out, lse, workspace, workspace_bytes, num_ctas, stream);
        if (st != PKV_OK || chunk_begin_out == nullptr || batch == 0) return st;
        cudaError_t e = cudaMemsetAsync(chunk_begin_out, 0, static_cast<size_t>(batch) * 4,
                                        as_stream(stream));
        return e == cudaSuccess ? PKV_OK : cuda_fail(e, "cudaMemsetAsync");
    }
    if (!(std::isfinite(sm_scale)))
        return fail(PKV_ERR_INVALID_ARG, "sm_scale must be finite");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and > 0");
    if (batch == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out || !lse)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 4) ||
        !aligned(lse, 4) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
        (chunk_begin_out && !aligned(chunk_begin_out, 4)))
        return fail(PKV_ERR_INVALID_ARG, "misaligned pointer (q and caches need 16 bytes)");
    if (!workspace || !aligned(workspace, 256))
        return fail(PKV_ERR_WORKSPACE, "workspace must be non-null and 256-byte aligned");

    AttnPlan plan;
    st = plan_attention(true, batch, num_kv_heads, group, head_dim, max_pages, page_size, num_ctas,
                        &plan, /*allow_cluster=*/false);
    if (st != PKV_OK) return st;
    const DeviceInfo* info = nullptr;
    st = device_info(&info);
    if (st != PKV_OK) return st;
    const pkv::WorkspaceLayout wl =
        pkv::workspace_layout(batch, group, num_kv_heads, 2, head_dim, plan.grid);
    const PrefixLayout pl = prefix_layout(wl.total, batch, num_kv_heads, group);
    if (workspace_bytes < pl.total)
        return fail(PKV_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes,
                    pl.total);
    int pfx_blocks = 1;   // resident shared-prefix CTAs per SM
    {
        static std::mutex m;
        static int blocks[kMaxDevices] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
        std::lock_guard<std::mutex> lock(m);
        if (blocks[dev] == 0) {
            e = pkv::prefix_set_smem_attr();
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
            int n = 0;
            e = pkv::prefix_occupancy(&n);
            if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
            if (n < 1) {
                int regs = 0, local = 0, maxt = 0;
                pkv::prefix_attributes(&regs, &local, &maxt);
                return fail(PKV_ERR_UNSUPPORTED,
                            "the shared-prefix kernel does not fit on an SM of this device "
                            "(%d registers, %d local bytes per thread, at most %d threads per CTA)",
                            regs, local, maxt);
            }
            blocks[dev] = n;
        }
        pfx_blocks = blocks[dev];
    }

    const int box_rows = page_size < pkv::kChunkTokens ? page_size : pkv::kChunkTokens;
    const int64_t rows = static_cast<int64_t>(num_pages) * num_kv_heads * page_size;
    CUtensorMap tk_p, tv_p, tk, tv;
    // the prefix pass loads one head's 64 rows (or a page of them) per box
    st = encode_pool_map(&tk_p, k_cache, true, head_dim, rows, box_rows);
    if (st != PKV_OK) return st;
    st = encode_pool_map(&tv_p, v_cache, true, head_dim, rows, box_rows);
    if (st != PKV_OK) return st;
    // the split-K kernel's boxes (both heads of a 64-token page at once)
    const int box_rows_s = page_size == pkv::kChunkTokens ? 2 * pkv::kChunkTokens : box_rows;
    st = encode_pool_map(&tk, k_cache, true, head_dim, rows, box_rows_s);
    if (st != PKV_OK) return st;
    st = encode_pool_map(&tv, v_cache, true, head_dim, rows, box_rows_s);
    if (st != PKV_OK) return st;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const float qk_scale = sm_scale * k_scale * 1.4426950408889634f;
    pkv::PrefixArgs pa{};
    pa.q = q;
    pa.page_table = page_table;
    pa.seq_lens = seq_lens;
    pa.abort = abort;
    pa.status = reinterpret_cast<uint32_t*>(ws);
    pa.pfx_ml = reinterpret_cast<float*>(ws + pl.pml_off);
    pa.pfx_o = reinterpret_cast<float*>(ws + pl.po_off);
    pa.link = reinterpret_cast<int32_t*>(ws + pl.link_off);
    pa.leader = reinterpret_cast<int32_t*>(ws + pl.leader_off);
    pa.refkey = reinterpret_cast<unsigned long long*>(ws + pl.refkey_off);
    pa.ref = reinterpret_cast<int32_t*>(ws + pl.ref_off);
    pa.share = reinterpret_cast<int32_t*>(ws + pl.share_off);
    pa.pshare = reinterpret_cast<int32_t*>(ws + pl.pshare_off);
    pa.chunk_begin = reinterpret_cast<int32_t*>(ws + pl.cbeg_off);
    pa.tiles = reinterpret_cast<int32_t*>(ws + pl.tiles_off);
    pa.num_tiles = reinterpret_cast<int32_t*>(ws + pl.ntiles_off);
    pa.batch = batch;
    pa.max_pages = max_pages;
    pa.num_q_heads = num_q_heads;
    pa.num_kv_heads = num_kv_heads;
    pa.group = group;
    pa.page_size = page_size;
    pa.num_pages = num_pages;
    pa.box_rows = box_rows;
    pa.items_per_req = num_kv_heads / 2;
    pa.members_per_tile = 64 / group;
    pa.min_chunks = pkv::kPfxMinChunks;
    pa.tail_chunks = pkv::kPfxTailChunks;
    pa.out = out;
    pa.lse = lse;
    pa.qk_scale = qk_scale;
    pa.v_scale = v_scale;

    cudaStream_t s = as_stream(stream);
    cudaError_t e = pkv::launch_prefix_plan(s, pa);
    if (e != cudaSuccess) return cuda_fail(e, "shared-prefix plan launch");
    // one wave of tile CTAs, each looping over the tiles
    e = pkv::launch_prefix_attn(pfx_blocks * info->sms, s, tk_p, tv_p, pa);
    if (e != cudaSuccess) return cuda_fail(e, "shared-prefix attention launch");

    pkv::AttnArgs a{};
    a.q = q;
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.abort = abort;
    a.out = out;
    a.lse = lse;
    a.ws_status = reinterpret_cast<uint32_t*>(ws);
    a.ws_ml = reinterpret_cast<float*>(ws + wl.ml_off);
    a.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
    a.batch = batch;
    a.max_pages = max_pages;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.kv_per_item = 2;
    a.items_per_req = num_kv_heads / 2;
    a.group = group;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.num_ctas = plan.grid;
    a.box_rows = box_rows_s;
    a.cluster_size = 0;
    a.num_clusters = 0;
    a.qk_scale = qk_scale;
    a.v_scale = v_scale;
    a.chunk_begin = pa.chunk_begin;
    a.pfx_ml = pa.pfx_ml;
    a.pfx_o = pa.pfx_o;
    e = pkv::launch_attn_partial(true, head_dim, group_pad_of(group), 2, plan.grid, s, tk, tv, a);
    if (e != cudaSuccess) return cuda_fail(e, "attention partial launch");
    e = pkv::launch_attn_merge(head_dim, s, a);
    if (e != cudaSuccess) return cuda_fail(e, "attention merge launch");
    if (chunk_begin_out != nullptr) {
        e = cudaMemcpyAsync(chunk_begin_out, pa.chunk_begin, static_cast<size_t>(batch) * 4,
                            cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync");
    }
    return PKV_OK;
}

}  // namespace

namespace pkv {
void set_last_error(const char* message) { g_last_error = message; }

WorkspaceLayout workspace_layout(int32_t batch, int32_t group, int32_t num_kv_heads,
                                 int32_t kv_per_item, int32_t head_dim, int32_t num_ctas) {
    WorkspaceLayout l{};
    const size_t items = static_cast<size_t>(batch) * (num_kv_heads / kv_per_item);
    const size_t heads_per_slot = static_cast<size_t>(group) * kv_per_item;
    const size_t slots = static_cast<size_t>(num_ctas) + items;
    l.ml_off = 256;   // after the status word
    l.o_off = round_up(l.ml_off + slots * heads_per_slot * 4 * 4, 256);
    l.total = round_up(l.o_off + slots * heads_per_slot * head_dim * 4, 256);
    return l;
}
}  // namespace pkv

extern "C" {

const char* pkv_last_error(void) { return g_last_error.c_str(); }

int32_t pkv_version(void) { return 100; }

pkv_status kv_tag_check(const uint32_t* page_tags, int32_t num_pages, const int32_t* page_table,
                        const uint32_t* expected_tags, int32_t max_pages, const int32_t* seq_lens,
                        int32_t batch, int32_t page_size, uint8_t* abort_out,
                        int32_t* num_aborted, void* stream) {
    if (batch < 0) return fail(PKV_ERR_INVALID_ARG, "batch must be >= 0");
    if (num_pages < 1 || max_pages < 1 || page_size < 1)
        return fail(PKV_ERR_INVALID_ARG, "num_pages, max_pages and page_size must be >= 1");
    if (batch > 0 && (!page_tags || !page_table || !expected_tags || !seq_lens || !abort_out))
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (num_aborted) {
        cudaError_t e = cudaMemsetAsync(num_aborted, 0, sizeof(int32_t), as_stream(stream));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(num_aborted)");
    }
    if (batch == 0) return PKV_OK;
    {
        const DeviceInfo* info = nullptr;   // per-device set-up (kernel attributes)
        const pkv_status ds = device_info(&info);
        if (ds != PKV_OK) return ds;
    }
    cudaError_t e = pkv::launch_tag_check(page_tags, num_pages, page_table, expected_tags,
                                          max_pages, seq_lens, batch, page_size, abort_out,
                                          num_aborted, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tag check launch");
    return PKV_OK;
}

static pkv_status append_impl(bool fp8, const uint16_t* k_new, const uint16_t* v_new,
                              const int32_t* page_table, int32_t max_pages,
                              const int32_t* seq_lens, int32_t batch, int32_t num_kv_heads,
                              int32_t head_dim, int32_t page_size, float k_scale, float v_scale,
                              void* k_cache, void* v_cache, int32_t num_pages,
                              const uint8_t* abort, void* stream) {
    pkv_status st = check_common_kv(batch, num_kv_heads, head_dim, page_size, num_pages, max_pages);
    if (st != PKV_OK) return st;
    if (fp8 && (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
                !std::isfinite(v_scale)))
        return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and > 0");
    if (batch == 0) return PKV_OK;
    if (!k_new || !v_new || !page_table || !seq_lens || !k_cache || !v_cache)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG, "k_new, v_new and the caches must be 16-byte aligned");
    {
        const DeviceInfo* info = nullptr;   // per-device set-up (kernel attributes)
        const pkv_status ds = device_info(&info);
        if (ds != PKV_OK) return ds;
    }
    cudaError_t e = pkv::launch_append(fp8, k_new, v_new, page_table, max_pages, seq_lens, batch,
                                       num_kv_heads, head_dim, page_size, k_scale, v_scale,
                                       k_cache, v_cache, num_pages, abort, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    return PKV_OK;
}

pkv_status kv_append_fp8(const uint16_t* k_new, const uint16_t* v_new, const int32_t* page_table,
                         int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                         int32_t num_kv_heads, int32_t head_dim, int32_t page_size, float k_scale,
                         float v_scale, uint8_t* k_cache, uint8_t* v_cache, int32_t num_pages,
                         const uint8_t* abort, void* stream) {
    return append_impl(true, k_new, v_new, page_table, max_pages, seq_lens, batch, num_kv_heads,
                       head_dim, page_size, k_scale, v_scale, k_cache, v_cache, num_pages, abort,
                       stream);
}

pkv_status kv_append_bf16(const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                          int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                          int32_t page_size, uint16_t* k_cache, uint16_t* v_cache,
                          int32_t num_pages, const uint8_t* abort, void* stream) {
    return append_impl(false, k_new, v_new, page_table, max_pages, seq_lens, batch, num_kv_heads,
                       head_dim, page_size, 1.f, 1.f, k_cache, v_cache, num_pages, abort, stream);
}

static pkv_status check_append_impl(bool fp8, const uint32_t* page_tags, int32_t num_pages,
                                    const int32_t* page_table, const uint32_t* expected_tags,
                                    int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                    int32_t page_size, const uint16_t* k_new,
                                    const uint16_t* v_new, int32_t num_kv_heads,
                                    int32_t head_dim, float k_scale, float v_scale, void* k_cache,
                                    void* v_cache, uint8_t* abort_out, int32_t* num_aborted,
                                    void* stream) {
    pkv_status st = check_common_kv(batch, num_kv_heads, head_dim, page_size, num_pages, max_pages);
    if (st != PKV_OK) return st;
    if (fp8 && (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
                !std::isfinite(v_scale)))
        return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and > 0");
    if (num_aborted) {
        cudaError_t e = cudaMemsetAsync(num_aborted, 0, sizeof(int32_t), as_stream(stream));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(num_aborted)");
    }
    if (batch == 0) return PKV_OK;
    if (!page_tags || !page_table || !expected_tags || !seq_lens || !k_new || !v_new ||
        !k_cache || !v_cache || !abort_out)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG, "k_new, v_new and the caches must be 16-byte aligned");
    {
        const DeviceInfo* info = nullptr;   // per-device set-up (kernel attributes)
        const pkv_status ds = device_info(&info);
        if (ds != PKV_OK) return ds;
    }
    cudaError_t e = pkv::launch_check_append(fp8, page_tags, num_pages, page_table, expected_tags,
                                             max_pages, seq_lens, batch, page_size, k_new, v_new,
                                             num_kv_heads, head_dim, k_scale, v_scale, k_cache,
                                             v_cache, abort_out, num_aborted, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "check+append launch");
    return PKV_OK;
}

pkv_status kv_check_append_fp8(const uint32_t* page_tags, int32_t num_pages,
                               const int32_t* page_table, const uint32_t* expected_tags,
                               int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                               int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                               int32_t num_kv_heads, int32_t head_dim, float k_scale,
                               float v_scale, uint8_t* k_cache, uint8_t* v_cache,
                               uint8_t* abort_out, int32_t* num_aborted, void* stream) {
    return check_append_impl(true, page_tags, num_pages, page_table, expected_tags, max_pages,
                             seq_lens, batch, page_size, k_new, v_new, num_kv_heads, head_dim,
                             k_scale, v_scale, k_cache, v_cache, abort_out, num_aborted, stream);
}

pkv_status kv_check_append_bf16(const uint32_t* page_tags, int32_t num_pages,
                                const int32_t* page_table, const uint32_t* expected_tags,
                                int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                                int32_t num_kv_heads, int32_t head_dim, uint16_t* k_cache,
                                uint16_t* v_cache, uint8_t* abort_out, int32_t* num_aborted,
                                void* stream) {
    return check_append_impl(false, page_tags, num_pages, page_table, expected_tags, max_pages,
                             seq_lens, batch, page_size, k_new, v_new, num_kv_heads, head_dim,
                             1.f, 1.f, k_cache, v_cache, abort_out, num_aborted, stream);
}

pkv_status kv_retag_pages(uint32_t* page_tags, int32_t num_pages, const int32_t* pages,
                          int32_t num_ids, void* stream) {
    if (num_pages < 1 || num_ids < 0)
        return fail(PKV_ERR_INVALID_ARG, "num_pages must be >= 1 and num_ids >= 0");
    if (num_ids == 0) return PKV_OK;
    if (!page_tags || !pages) return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(page_tags, 4) || !aligned(pages, 4))
        return fail(PKV_ERR_INVALID_ARG, "misaligned pointer");
    cudaError_t e = pkv::launch_retag(page_tags, num_pages, pages, num_ids, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "retag launch");
    return PKV_OK;
}

pkv_status kv_expected_tags(const uint32_t* page_tags, int32_t num_pages,
                            const int32_t* page_table, int32_t max_pages,
                            const int32_t* seq_lens, int32_t batch, int32_t page_size,
                            uint32_t* expected_tags, void* stream) {
    if (batch < 0 || num_pages < 1 || max_pages < 1 || page_size < 1)
        return fail(PKV_ERR_INVALID_ARG, "invalid sizes");
    if (batch == 0) return PKV_OK;
    if (!page_tags || !page_table || !seq_lens || !expected_tags)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    cudaError_t e = pkv::launch_expected_tags(page_tags, num_pages, page_table, max_pages,
                                              seq_lens, batch, page_size, expected_tags,
                                              as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "expected-tags launch");
    return PKV_OK;
}

pkv_status kv_requant_pages_fp8(const uint16_t* src_pool, int32_t src_num_pages,
                                const int32_t* src_pages, uint8_t* dst_pool,
                                int32_t dst_num_pages, const int32_t* dst_pages,
                                int32_t num_pairs, int32_t num_kv_heads, int32_t page_size,
                                int32_t head_dim, float scale, void* stream) {
    if (num_pairs < 0) return fail(PKV_ERR_INVALID_ARG, "num_pairs must be >= 0");
    if (src_num_pages < 1 || dst_num_pages < 1 || num_kv_heads < 1)
        return fail(PKV_ERR_INVALID_ARG, "pool sizes and num_kv_heads must be >= 1");
    if (!supported_head_dim(head_dim))
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
    if (!supported_page_size(page_size))
        return fail(PKV_ERR_UNSUPPORTED, "page_size %d not supported", page_size);
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(PKV_ERR_INVALID_ARG, "scale must be finite and > 0");
    if (num_pairs == 0) return PKV_OK;
    if (!src_pool || !src_pages || !dst_pool || !dst_pages)
        return fail(PKV_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned(src_pool, 16) || !aligned(dst_pool, 16))
        return fail(PKV_ERR_INVALID_ARG, "pools must be 16-byte aligned");
    const int64_t page_elems = static_cast<int64_t>(num_kv_heads) * page_size * head_dim;
    cudaError_t e = pkv::launch_requant(src_pool, src_num_pages, src_pages, dst_pool,
                                        dst_num_pages, dst_pages, num_pairs, page_elems, scale,
                                        as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "requant launch");
    return PKV_OK;
}

pkv_status paged_decode_attn_plan(int32_t kv_dtype, int32_t batch, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim, int32_t max_pages,
                                  int32_t page_size, int32_t num_ctas, int32_t* cluster_size,
                                  int32_t* ctas, int32_t* launches) {
    if (kv_dtype != PKV_KV_FP8 && kv_dtype != PKV_KV_BF16)
        return fail(PKV_ERR_INVALID_ARG, "kv_dtype must be PKV_KV_FP8 or PKV_KV_BF16");
    if (!cluster_size || !ctas || !launches)
        return fail(PKV_ERR_INVALID_ARG, "null output pointer");
    if (batch < 1) return fail(PKV_ERR_INVALID_ARG, "batch must be >= 1");
    pkv_status st = check_common_kv(batch, num_kv_heads, head_dim, page_size, 1, max_pages);
    if (st != PKV_OK) return st;
    if (num_q_heads < 1 || num_q_heads % num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
    const int group = num_q_heads / num_kv_heads;
    if (group > 16) return fail(PKV_ERR_UNSUPPORTED, "GQA group %d > 16 not supported", group);
    if (num_ctas < -pkv::kMaxCluster)
        return fail(PKV_ERR_INVALID_ARG, "num_ctas must be >= %d", -pkv::kMaxCluster);
    AttnPlan plan;
    st = plan_attention(kv_dtype == PKV_KV_FP8, batch, num_kv_heads, group, head_dim, max_pages,
                        page_size, num_ctas, &plan);
    if (st != PKV_OK) return st;
    *cluster_size = plan.cluster;
    *ctas = plan.cluster > 0 ? plan.cluster * plan.nclusters : plan.grid;
    *launches = plan.cluster > 0 ? 1 : 2;
    return PKV_OK;
}

size_t paged_decode_attn_workspace_size(int32_t kv_dtype, int32_t batch, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim,
                                        int32_t num_ctas) {
    if (kv_dtype != PKV_KV_FP8 && kv_dtype != PKV_KV_BF16) {
        fail(PKV_ERR_INVALID_ARG, "kv_dtype must be PKV_KV_FP8 or PKV_KV_BF16");
        return 0;
    }
    if (batch < 0 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
        !supported_head_dim(head_dim) || num_ctas < -pkv::kMaxCluster) {
        fail(PKV_ERR_INVALID_ARG, "invalid sizes for the workspace query");
        return 0;
    }
    const int group = num_q_heads / num_kv_heads;
    if (group > 16) {
        fail(PKV_ERR_UNSUPPORTED, "GQA group %d > 16 not supported", group);
        return 0;
    }
    int grid = num_ctas > 0 ? num_ctas : 0;   // cluster mode (< 0) needs no more than the default
    const bool fp8 = kv_dtype == PKV_KV_FP8;
    const int kv_per_item = pkv::kv_heads_per_item(fp8, num_kv_heads, group);
    if (grid == 0 && default_ctas(fp8, head_dim, group, kv_per_item, &grid) != PKV_OK) return 0;
    return pkv::workspace_layout(batch, group, num_kv_heads, kv_per_item, head_dim, grid).total;
}

pkv_status paged_decode_attn_fp8(const uint16_t* q, const uint8_t* k_cache,
                                 const uint8_t* v_cache, float k_scale, float v_scale,
                                 const int32_t* page_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                                 int32_t num_pages, float sm_scale, const uint8_t* abort,
                                 uint16_t* out, float* lse, void* workspace,
                                 size_t workspace_bytes, int32_t num_ctas, void* stream) {
    return attn_impl(true, q, k_cache, v_cache, k_scale, v_scale, page_table, max_pages, seq_lens,
                     batch, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, sm_scale,
                     abort, out, lse, workspace, workspace_bytes, num_ctas, stream);
}

size_t paged_decode_attn_fp8_prefix_workspace_size(int32_t batch, int32_t num_q_heads,
                                                   int32_t num_kv_heads, int32_t head_dim,
                                                   int32_t num_ctas) {
    if (batch < 0 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
        !supported_head_dim(head_dim) || num_ctas < 0) {
        fail(PKV_ERR_INVALID_ARG, "invalid sizes for the shared-prefix workspace query");
        return 0;
    }
    const int group = num_q_heads / num_kv_heads;
    if (!prefix_supported(num_kv_heads, group, head_dim))
        return paged_decode_attn_workspace_size(PKV_KV_FP8, batch, num_q_heads, num_kv_heads,
                                                head_dim, num_ctas);
    int grid = num_ctas;
    if (grid == 0 && default_ctas(true, head_dim, group, 2, &grid) != PKV_OK) return 0;
    const size_t base = pkv::workspace_layout(batch, group, num_kv_heads, 2, head_dim, grid).total;
    return prefix_layout(base, batch, num_kv_heads, group).total;
}

pkv_status paged_decode_attn_fp8_prefix(const uint16_t* q, const uint8_t* k_cache,
                                        const uint8_t* v_cache, float k_scale, float v_scale,
                                        const int32_t* page_table, int32_t max_pages,
                                        const int32_t* seq_lens, int32_t batch,
                                        int32_t num_q_heads, int32_t num_kv_heads,
                                        int32_t head_dim, int32_t page_size, int32_t num_pages,
                                        float sm_scale, const uint8_t* abort, uint16_t* out,
                                        float* lse, void* workspace, size_t workspace_bytes,
                                        int32_t num_ctas, int32_t* chunk_begin_out,
                                        void* stream) {
    return prefix_impl(q, k_cache, v_cache, k_scale, v_scale, page_table, max_pages, seq_lens,
                       batch, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, sm_scale,
                       abort, out, lse, workspace, workspace_bytes, num_ctas, chunk_begin_out,
                       stream);
}

pkv_status paged_decode_attn_bf16(const uint16_t* q, const uint16_t* k_cache,
                                  const uint16_t* v_cache, const int32_t* page_table,
                                  int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t page_size, int32_t num_pages, float sm_scale,
                                  const uint8_t* abort, uint16_t* out, float* lse,
                                  void* workspace, size_t workspace_bytes, int32_t num_ctas,
                                  void* stream) {
    return attn_impl(false, q, k_cache, v_cache, 1.f, 1.f, page_table, max_pages, seq_lens, batch,
                     num_q_heads, num_kv_heads, head_dim, page_size, num_pages, sm_scale, abort,
                     out, lse, workspace, workspace_bytes, num_ctas, stream);
}

pkv_status int4_dequant_gemv(const uint16_t* x, const uint8_t* w_tiles, const uint16_t* scales,
                             int32_t batch, int32_t n, int32_t k, int32_t group_size, uint16_t* y,
                             uint32_t* status, void* stream) {
    if (!x || !w_tiles || !scales || !y)
        return fail(PKV_ERR_INVALID_ARG, "x, w_tiles, scales and y must be non-null");
    if (!aligned(x, 16) || !aligned(w_tiles, 16) || !aligned(scales, 16) || !aligned(y, 2) ||
        (status && !aligned(status, 4)))
        return fail(PKV_ERR_INVALID_ARG,
                    "misaligned pointer (x, w_tiles and scales need 16 bytes, y 2, status 4)");
    if (batch < 1 || batch > pkv::kGemvMaxBatch)
        return fail(PKV_ERR_INVALID_ARG, "batch must be in [1, %d] (got %d)", pkv::kGemvMaxBatch,
                    batch);
    if (n < pkv::kGemvRows || n % pkv::kGemvRows != 0)
        return fail(PKV_ERR_INVALID_ARG, "n must be a positive multiple of %d (got %d)",
                    pkv::kGemvRows, n);
    if (k < pkv::kGemvKTile || k % pkv::kGemvKTile != 0)
        return fail(PKV_ERR_INVALID_ARG, "k must be a positive multiple of %d (got %d)",
                    pkv::kGemvKTile, k);
    if (group_size != pkv::kGemvGroup)
        return fail(PKV_ERR_UNSUPPORTED, "group_size %d not supported (%d)", group_size,
                    pkv::kGemvGroup);

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    // batches up to 16 on the warp-level MMA kernel, larger ones on tcgen05
    const bool small = batch <= pkv::kGemvMmaMaxBatch;
    const int xrows = small ? 8 * pkv::gemv_mma_batch_blocks(batch) : pkv::gemv_batch_cols(batch);
    {
        static std::mutex m;
        static bool ready[kMaxDevices][5] = {};
        const int slot = small ? (xrows == 8 ? 0 : 1) : (xrows == 16 ? 2 : (xrows == 32 ? 3 : 4));
        if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device %d", dev);
        std::lock_guard<std::mutex> lock(m);
        if (!ready[dev][slot]) {
            e = small ? pkv::gemv_mma_set_smem_attr(xrows / 8) : pkv::gemv_set_smem_attr(xrows);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
            ready[dev][slot] = true;
        }
    }

    // codes: the tiles as rows of 128 bytes (one box = one 128 x 256 tile);
    // x: [batch][k] bf16, 64-column x xrows-row boxes (rows past batch read
    // as zero); scales: rows of 128 (one row block, one group), 2-row boxes
    CUtensorMap tw, tx, ts;
    pkv_status st = encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_tiles, pkv::kGemvKTile / 2,
                              static_cast<uint64_t>(n) * (k / pkv::kGemvKTile),
                              pkv::kGemvKTile / 2, pkv::kGemvKTile / 2, pkv::kGemvRows,
                              CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != PKV_OK) return st;
    st = encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(k),
                   static_cast<uint64_t>(batch), static_cast<uint64_t>(k) * 2, 64, xrows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != PKV_OK) return st;
    st = encode_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales, pkv::kGemvRows,
                   static_cast<uint64_t>(n / pkv::kGemvRows) * (k / group_size),
                   pkv::kGemvRows * 2, pkv::kGemvRows, pkv::kGemvKTile / pkv::kGemvGroup,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != PKV_OK) return st;

    pkv::GemvArgs a{};
    a.y = y;
    a.status = status;
    a.batch = batch;
    a.n = n;
    a.k = k;
    e = small ? pkv::launch_int4_gemv_mma(xrows / 8, as_stream(stream), tw, tx, ts, a)
              : pkv::launch_int4_gemv(xrows, as_stream(stream), tw, tx, ts, a);
    if (e != cudaSuccess) return cuda_fail(e, "int4_dequant_gemv launch");
    return PKV_OK;
}

}  // extern "C"
