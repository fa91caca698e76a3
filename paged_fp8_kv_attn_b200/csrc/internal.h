// internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pkv {

// Tokens per pipeline stage of the attention kernels (one "chunk").
constexpr int kChunkTokens = 64;
// Largest thread-block cluster of the attention kernel's cluster mode (16 is
// the non-portable maximum on sm_100).
constexpr int kMaxCluster = 16;

// Arguments of the split-K partial and merge kernels (passed by value).
struct AttnArgs {
    const uint16_t* q;          // [B][Hq][D] bf16
    const int32_t* page_table;  // [B][MP]
    const int32_t* seq_lens;    // [B]
    const uint8_t* abort;       // [B] or null
    uint16_t* out;              // [B][Hq][D] bf16
    float* lse;                 // [B][Hq]
    uint32_t* ws_status;        // workspace word 0 (cleared by CTA 0 of each call)
    float* ws_ml;               // [slots][G][4]  (running max in log2 units, sum of the
                                //  fp32 weights, sum of the rounded weights, unused)
    float* ws_o;                // [slots][G][D]  (unnormalised, V scale applied)
    int32_t batch;
    int32_t max_pages;
    int32_t num_q_heads;
    int32_t num_kv_heads;       // KV heads of the pool
    int32_t kv_per_item;        // KV heads one work item covers (1 or 2)
    int32_t items_per_req;      // num_kv_heads / kv_per_item
    int32_t group;              // query heads per KV head
    int32_t page_size;
    int32_t num_pages;
    int32_t num_ctas;
    int32_t box_rows;           // rows per TMA box = min(page_size, 64)
    int32_t cluster_size;       // 0: split-K over the grid + merge kernel;
                                // C > 0: clusters of C CTAs, no merge kernel
    int32_t num_clusters;       // cluster mode: clusters in the grid
    float qk_scale;             // sm_scale * k_scale * log2(e)
    float v_scale;              // per-tensor V scale (1 for BF16)
    // Shared-prefix mode (all null otherwise): the split-K kernels cover
    // chunks [chunk_begin[b], n_b) of request b; the shared-prefix pass left
    // one record per item of the requests with chunk_begin[b] > 0, which the
    // merge kernel adds to the item's own records.
    const int32_t* chunk_begin;  // [B]
    const float* pfx_ml;         // [items][G][4]
    const float* pfx_o;          // [items][G][D]
};

// Shared-prefix pass (prefix.cu): FP8, head_dim 128, two KV heads per item.
constexpr int kPfxRows = 128;         // rows of one tensor-core tile (query heads of its members)
constexpr int kPfxRowThreads = 256;   // two threads per tile row
constexpr int kPfxThreads = 2 * (kPfxRowThreads + 32);   // two halves of 8 row warps + 1 TMA warp
constexpr int kPfxPlanThreads = 1024;
constexpr int kPfxMinChunks = 4;      // shared chunks that make a request join a group
constexpr int kPfxTailChunks = 2;     // own chunks a tile finishes for a member

struct PrefixArgs {
    const uint16_t* q;          // [B][Hq][128] bf16
    const int32_t* page_table;  // [B][MP]
    const int32_t* seq_lens;    // [B]
    const uint8_t* abort;       // [B] or null
    uint32_t* status;           // workspace status word
    float* pfx_ml;              // [items][2G][4]
    float* pfx_o;               // [items][2G][128]
    int32_t* link;              // [B]  shared chunks with request b - 1
    int32_t* leader;            // [B]  first request of b's group
    unsigned long long* refkey; // [B]  per group leader: (full chunks + 1, ~index) of its reference
    int32_t* ref;               // [B]  the reference row of b's group
    int32_t* share;             // [B]  shared chunks with the reference row
    int32_t* pshare;            // [B]  chunks the shared pass covers for b's rows
    int32_t* chunk_begin;       // [B]  first chunk of the split-K kernels (n_b: none left)
    int32_t* tiles;             // [B / 2 + 1][4]: page-table row, first member, members, chunks
    int32_t* num_tiles;         // [1]
    int32_t batch;
    int32_t max_pages;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t group;
    int32_t page_size;
    int32_t num_pages;
    int32_t box_rows;           // min(page_size, 64)
    int32_t items_per_req;      // num_kv_heads / 2
    int32_t members_per_tile;   // 64 / group
    int32_t min_chunks;
    int32_t tail_chunks;        // a member with at most this many chunks after its shared
                                // ones is finished by its tile (final outputs, no merge)
    float qk_scale;             // sm_scale * k_scale * log2(e)
    float v_scale;
    uint16_t* out;              // [B][Hq][128] bf16 (members the tile finishes)
    float* lse;                 // [B][Hq]
};
size_t prefix_attn_smem_bytes();
cudaError_t prefix_set_smem_attr();
cudaError_t prefix_occupancy(int* blocks_per_sm);
cudaError_t prefix_attributes(int* regs, int* local_bytes, int* max_threads);
// the plan kernels (two launches)
cudaError_t launch_prefix_plan(cudaStream_t stream, const PrefixArgs& args);
cudaError_t launch_prefix_attn(int grid, cudaStream_t stream, const CUtensorMap& tmap_k,
                               const CUtensorMap& tmap_v, const PrefixArgs& args);

// Sets the message pkv_last_error() returns on this thread.
void set_last_error(const char* message);

// KV heads one attention work item covers: two adjacent heads (one
// contiguous 16 KiB K or V block per 64-token page) for FP8 caches with an
// even number of KV heads and a GQA group of at most 8; otherwise one.
inline int kv_heads_per_item(bool fp8, int num_kv_heads, int group) {
    return (fp8 && num_kv_heads % 2 == 0 && group <= 8) ? 2 : 1;
}

// Workspace layout for given sizes and grid (slots = grid + work items).
struct WorkspaceLayout {
    size_t ml_off, o_off, total;
};
WorkspaceLayout workspace_layout(int32_t batch, int32_t group, int32_t num_kv_heads,
                                 int32_t kv_per_item, int32_t head_dim, int32_t num_ctas);

// Attention variant properties: dynamic shared memory bytes.  Returns 0 if
// the combination is not compiled.
size_t attn_partial_smem_bytes(bool fp8, int head_dim, int group_pad, int kv_per_item);
cudaError_t attn_set_smem_attr(bool fp8, int head_dim, int group_pad, int kv_per_item);
cudaError_t attn_occupancy(bool fp8, int head_dim, int group_pad, int kv_per_item,
                           int* blocks_per_sm);
constexpr int kAttnThreads = 160;   // 4 consumer warps + 1 producer warp

// Clusters of `cluster_size` CTAs that can be resident at once (0 if none).
cudaError_t attn_max_clusters(bool fp8, int head_dim, int group_pad, int kv_per_item,
                              int cluster_size, int* clusters);
// grid CTAs; with args.cluster_size > 0 launched as clusters of that size.
cudaError_t launch_attn_partial(bool fp8, int head_dim, int group_pad, int kv_per_item, int grid,
                                cudaStream_t stream, const CUtensorMap& tmap_k,
                                const CUtensorMap& tmap_v, const AttnArgs& args);
cudaError_t launch_attn_merge(int head_dim, cudaStream_t stream, const AttnArgs& args);

cudaError_t launch_tag_check(const uint32_t* page_tags, int32_t num_pages,
                             const int32_t* page_table, const uint32_t* expected_tags,
                             int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                             int32_t page_size, uint8_t* abort_out, int32_t* num_aborted,
                             cudaStream_t stream);

cudaError_t launch_append(bool fp8, const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                          int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                          int32_t page_size, float k_scale, float v_scale, void* k_cache,
                          void* v_cache, int32_t num_pages, const uint8_t* abort,
                          cudaStream_t stream);

// all of the SM's on-chip memory as shared memory for the step's first kernels
cudaError_t step_kernels_set_carveout();
cudaError_t launch_check_append(bool fp8, const uint32_t* page_tags, int32_t num_pages,
                                const int32_t* page_table, const uint32_t* expected_tags,
                                int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                                int32_t num_kv_heads, int32_t head_dim, float k_scale,
                                float v_scale, void* k_cache, void* v_cache, uint8_t* abort_out,
                                int32_t* num_aborted, cudaStream_t stream);

cudaError_t launch_retag(uint32_t* page_tags, int32_t num_pages, const int32_t* pages, int32_t n,
                         cudaStream_t stream);
cudaError_t launch_expected_tags(const uint32_t* page_tags, int32_t num_pages,
                                 const int32_t* page_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t batch, int32_t page_size,
                                 uint32_t* expected_tags, cudaStream_t stream);

cudaError_t launch_requant(const uint16_t* src_pool, int32_t src_num_pages,
                           const int32_t* src_pages, uint8_t* dst_pool, int32_t dst_num_pages,
                           const int32_t* dst_pages, int32_t num_pairs, int64_t page_elems,
                           float scale, cudaStream_t stream);

// INT4 weight dequantisation GEMV: CTA tile (weight rows), k-tile (columns
// per pipeline stage), scale group and largest batch.
constexpr int kGemvRows = 128;
constexpr int kGemvKTile = 256;
constexpr int kGemvGroup = 128;
constexpr int kGemvMaxBatch = 64;

struct GemvArgs {
    uint16_t* y;          // [batch][n] bf16
    uint32_t* status;     // nullable: bit 0 set if a bounded wait expired
    int32_t batch;
    int32_t n;
    int32_t k;
};

// Batches up to kGemvMmaMaxBatch run on the warp-level MMA kernel
// (int4_gemv_mma.cu), larger ones on the tcgen05 kernel (int4_gemv.cu).
constexpr int kGemvMmaMaxBatch = 16;

// tcgen05 kernel: batch columns of the tensor-core tile (16, 32 or 64).
int gemv_batch_cols(int batch);
cudaError_t gemv_set_smem_attr(int ncols);
// warp-level MMA kernel: batch blocks of 8 (1 or 2).
int gemv_mma_batch_blocks(int batch);
cudaError_t gemv_mma_set_smem_attr(int nb);
cudaError_t launch_int4_gemv_mma(int nb, cudaStream_t stream, const CUtensorMap& tmap_w,
                                 const CUtensorMap& tmap_x, const CUtensorMap& tmap_s,
                                 const GemvArgs& args);
cudaError_t launch_int4_gemv(int ncols, cudaStream_t stream, const CUtensorMap& tmap_w,
                             const CUtensorMap& tmap_x, const CUtensorMap& tmap_s,
                             const GemvArgs& args);

// Launch configuration with the programmatic-stream-serialisation attribute
// (and, optionally, a 1-D thread-block cluster shape).
struct PdlLaunch {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t stream) {
        cfg = cudaLaunchConfig_t{};
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    void set_cluster(int size) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(size);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
};

}  // namespace pkv
