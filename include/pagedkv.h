/*
 * pagedkv.h -- C ABI of the paged FP8-KV decode library for NVIDIA B200
 * (sm_100a).
 *
 * The calls follow the problem as the source pages state it: a pool of
 * physical KV-cache pages; per request a page table (logical page ->
 * physical page); per page a uint32 tag that changes whenever the page is
 * reallocated; per request the tags it expects; and a check, run as a
 * separate batched step before a supported decode op reads the cache, that
 * aborts any request whose page table names a page whose tag no longer
 * matches.  Pages cited below:
 *   [T] "大模型推理优化：量化、压缩与安全验证" (Chinese translation of the
 *       first-party post), sections "量化 KV cache" and "保护共享 KV cache";
 *   [S] siami.tw editorial on Cloudflare's Kimi/GLM inference, sections
 *       "KV 快取量化" (Table 1) and "共享 KV 快取的完整性檢查" (Table 3);
 *   [R] remio.ai commentary "Cloudflare 小型模型服务降低内存占用，但安全性成为考验",
 *       section "共享 KV 缓存安全性成为生产问题".
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Memory: every array argument is DEVICE memory owned by the caller.  The
 *    library allocates nothing, frees nothing and keeps no per-call state;
 *    its only state is a thread-local error string and a per-device cache of
 *    launch limits.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t); FP8 values
 *    are E4M3 codes (uint8_t): 1 sign bit, 4 exponent bits with bias 7,
 *    3 mantissa bits, S.1111.111 = NaN, no infinities, largest value 448.
 *  - KV pools are laid out [num_pages][num_kv_heads][page_size][head_dim],
 *    so one (page, KV head) tile is contiguous.  K and V live in separate
 *    pools of the same shape.
 *  - page_table and expected_tags are [batch][max_pages] (row stride
 *    max_pages); only the first ceil(seq_lens[b] / page_size) entries of a
 *    row are ever read.
 *  - seq_lens[b] counts the request's new token: the new token sits at
 *    position seq_lens[b] - 1.
 *  - abort is a [batch] uint8 mask (nonzero = aborted); it may be NULL
 *    wherever it is an input, meaning "no request is aborted" (the
 *    integrity check switched off; [T] "保护共享 KV cache": the default path
 *    is a no-op tracker with no measurable cost).
 *  - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *    Every call only enqueues work: it returns before the GPU runs it, and
 *    never synchronises.
 *  - Launch chaining: every kernel is launched with programmatic dependent
 *    launch, so it may be scheduled while the previous kernel on the stream
 *    is still running.  Each kernel
 *    waits for that kernel to finish before it touches memory that kernel
 *    may write, with one exception documented at paged_decode_attn_fp8:
 *    before waiting, attention reads q, seq_lens and page_table and
 *    prefetches K/V pages into L2 (nothing it reads before the wait reaches
 *    its outputs).
 *  - Errors: a status code is returned.  Invalid arguments are detected on
 *    the host before anything is enqueued (PKV_ERR_INVALID_ARG,
 *    PKV_ERR_WORKSPACE, PKV_ERR_UNSUPPORTED); a failed launch returns
 *    PKV_ERR_CUDA.  pkv_last_error() describes the last non-OK status on the
 *    calling thread.  Bad DEVICE data never traps a kernel: a page id outside
 *    [0, num_pages) or a length outside [1, max_pages * page_size] makes the
 *    request behave as aborted.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t pkv_status;
#define PKV_OK 0
#define PKV_ERR_INVALID_ARG 1   /* bad pointer, size, shape or alignment   */
#define PKV_ERR_WORKSPACE 2     /* workspace missing or too small          */
#define PKV_ERR_UNSUPPORTED 3   /* valid but not implemented (e.g. D=96)   */
#define PKV_ERR_CUDA 4          /* a CUDA runtime call or launch failed     */

#define PKV_KV_FP8 0
#define PKV_KV_BF16 1

/* Supported shapes: head_dim in {64, 128}; page_size in {16, 32, 64, 128};
 * num_q_heads a multiple of num_kv_heads with a group of at most 16;
 * num_pages * num_kv_heads * page_size < 2^31. */

/*
 * kv_tag_check -- batched page-tag integrity check.
 * [T] "保护共享 KV cache"; [S] "共享 KV 快取的完整性檢查"; [R] "共享 KV 缓存安全性成为生产问题":
 * each physical page has a tag that changes on reallocation; the server
 * records each request's expected pages and tags; before a supported decode
 * op reads the cache the mapping is checked, and a mismatching request is
 * aborted instead of returning data from the wrong page.  The check is its
 * own batched kernel, not fused into attention ([S] Table 3 discussion).
 *
 * For each request b:
 *   abort_out[b] = 1 if seq_lens[b] is outside [1, max_pages * page_size], or
 *   if some entry j < ceil(seq_lens[b] / page_size) has page_table[b][j]
 *   outside [0, num_pages) or page_tags[page_table[b][j]] !=
 *   expected_tags[b][j]; otherwise 0.  Every abort_out[b] is written.
 *   Entries past the used ones are never read.
 * page_tags [num_pages] uint32; page_table [batch][max_pages] int32;
 * expected_tags [batch][max_pages] uint32; seq_lens [batch] int32;
 * abort_out [batch] uint8 (written); num_aborted: NULL or one int32 that
 * receives the number of aborted requests (it is zeroed on the stream first).
 */
PKV_API pkv_status kv_tag_check(const uint32_t* page_tags, int32_t num_pages,
                        const int32_t* page_table, const uint32_t* expected_tags,
                        int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                        int32_t page_size, uint8_t* abort_out, int32_t* num_aborted,
                        void* stream);

/*
 * kv_append_fp8 -- quantise each request's new K/V token to E4M3 and write
 * it into its physical page.  [T] "量化 KV cache" / [S] "KV 快取量化": the KV
 * cache is stored as FP8 e4m3, halving it against BF16.
 *
 * For request b with L = seq_lens[b] and pos = L - 1, every element x of
 * k_new[b] (resp. v_new[b]) is written to
 *   k_cache[page_table[b][pos / page_size]][h][pos % page_size][d]
 * as the E4M3 code of y = x / k_scale, where y is the correctly rounded
 * binary32 quotient and the code is y rounded to nearest, ties to even,
 * with |y| > 448 (Inf included) saturated to +-448, a NaN x written as
 * S.1111.111 with the sign bit of x, and signed zeros kept.
 * Requests with abort[b] != 0 (abort may be NULL), a length outside
 * [1, max_pages * page_size] or a page id outside [0, num_pages) are
 * skipped.  k_new, v_new: [batch][num_kv_heads][head_dim] bf16, 16-byte
 * aligned.  k_scale, v_scale: finite and > 0 (per-tensor scales).
 */
PKV_API pkv_status kv_append_fp8(const uint16_t* k_new, const uint16_t* v_new,
                         const int32_t* page_table, int32_t max_pages,
                         const int32_t* seq_lens, int32_t batch, int32_t num_kv_heads,
                         int32_t head_dim, int32_t page_size, float k_scale, float v_scale,
                         uint8_t* k_cache, uint8_t* v_cache, int32_t num_pages,
                         const uint8_t* abort, void* stream);

/*
 * kv_append_bf16 -- the same write for a BF16 cache (the value is stored
 * unchanged).  The BF16 cache is the comparison point of [S] Table 1.
 */
PKV_API pkv_status kv_append_bf16(const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* page_table, int32_t max_pages,
                          const int32_t* seq_lens, int32_t batch, int32_t num_kv_heads,
                          int32_t head_dim, int32_t page_size,
                          uint16_t* k_cache, uint16_t* v_cache, int32_t num_pages,
                          const uint8_t* abort, void* stream);

/*
 * kv_check_append_fp8 -- kv_tag_check followed by kv_append_fp8 (with the
 * abort mask just computed), as one kernel with one CTA per request.
 * [T] "保护共享 KV cache" / [S] "共享 KV 快取的完整性檢查": the check stays a
 * batched pass of its own, separate from the attention kernel; only the
 * append, whose write of request b depends on nothing but request b's own
 * check, rides along.  Outputs are exactly those of the two calls in
 * sequence: abort_out[b] and num_aborted as kv_tag_check defines them, and
 * the new token of every request that passed written as kv_append_fp8
 * defines it.  Arguments: the union of the two calls' arguments, with the
 * same meaning, layout and alignment rules.
 */
PKV_API pkv_status kv_check_append_fp8(const uint32_t* page_tags, int32_t num_pages,
                               const int32_t* page_table, const uint32_t* expected_tags,
                               int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                               int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                               int32_t num_kv_heads, int32_t head_dim, float k_scale,
                               float v_scale, uint8_t* k_cache, uint8_t* v_cache,
                               uint8_t* abort_out, int32_t* num_aborted, void* stream);

/* kv_check_append_bf16 -- the same for a BF16 cache (kv_append_bf16). */
PKV_API pkv_status kv_check_append_bf16(const uint32_t* page_tags, int32_t num_pages,
                                const int32_t* page_table, const uint32_t* expected_tags,
                                int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                                int32_t num_kv_heads, int32_t head_dim, uint16_t* k_cache,
                                uint16_t* v_cache, uint8_t* abort_out, int32_t* num_aborted,
                                void* stream);

/*
 * kv_retag_pages -- device-side tag bump for reallocated pages.
 * [T] "保护共享 KV cache": a physical page gets a tag that changes whenever the
 * page is reallocated; [R] "共享 KV 缓存安全性成为生产问题" likens it to a
 * generation counter.  For every i < num_ids with pages[i] inside
 * [0, num_pages): page_tags[pages[i]] += 1 (mod 2^32), once per occurrence in
 * the list (atomically, so duplicates are counted).  Other ids are ignored.
 * page_tags [num_pages] uint32 (updated in place); pages [num_ids] int32.
 */
PKV_API pkv_status kv_retag_pages(uint32_t* page_tags, int32_t num_pages, const int32_t* pages,
                                  int32_t num_ids, void* stream);

/*
 * kv_expected_tags -- rebuild each request's expected tags from the current
 * page tags ([T] "保护共享 KV cache": the server records the pages and tags each
 * request expects).  For every request b with seq_lens[b] inside
 * [1, max_pages * page_size] and every used entry j < ceil(seq_lens[b] /
 * page_size) naming a page inside [0, num_pages):
 *   expected_tags[b][j] = page_tags[page_table[b][j]].
 * Every other entry is left unchanged.  Layouts as for kv_tag_check.
 */
PKV_API pkv_status kv_expected_tags(const uint32_t* page_tags, int32_t num_pages,
                                    const int32_t* page_table, int32_t max_pages,
                                    const int32_t* seq_lens, int32_t batch, int32_t page_size,
                                    uint32_t* expected_tags, void* stream);

/*
 * kv_requant_pages_fp8 -- BF16 -> FP8 page handoff.  [S] "KV 快取量化" and
 * [T] "量化 KV cache": the prefill pool keeps a BF16 cache while the decode
 * pool stores FP8.  Page src_pages[i] of the BF16 pool is re-quantised into
 * page dst_pages[i] of the FP8 pool, element by element with exactly the
 * rounding of kv_append_fp8.  Pairs naming an id outside their pool are
 * skipped.  src_pool [src_num_pages][Hkv][P][D] bf16; dst_pool
 * [dst_num_pages][Hkv][P][D] uint8; src_pages, dst_pages [num_pairs] int32.
 * Call once for K (with k_scale) and once for V (with v_scale).
 */
PKV_API pkv_status kv_requant_pages_fp8(const uint16_t* src_pool, int32_t src_num_pages,
                                const int32_t* src_pages, uint8_t* dst_pool,
                                int32_t dst_num_pages, const int32_t* dst_pages,
                                int32_t num_pairs, int32_t num_kv_heads, int32_t page_size,
                                int32_t head_dim, float scale, void* stream);

/*
 * paged_decode_attn_workspace_size -- bytes of device workspace the
 * attention calls need for these sizes.  kv_dtype is PKV_KV_FP8 or
 * PKV_KV_BF16; num_ctas is the value passed to the attention call (0 = the
 * default; > 0 a split-K grid of that many CTAs; -C, C in 1..16, cluster
 * mode, which needs no more than the default).  Returns 0 on invalid
 * arguments (see pkv_last_error).  The
 * workspace holds a status word and the split-K partial results.  Its
 * first 4 bytes are a status word that every
 * attention call writes: 0, or 1 if an internal bounded wait expired in that
 * call (never expected; the outputs are then unreliable).  The caller may
 * read it once the stream has finished the call.
 */
PKV_API size_t paged_decode_attn_workspace_size(int32_t kv_dtype, int32_t batch, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim,
                                        int32_t num_ctas);

/*
 * paged_decode_attn_plan -- the work split that paged_decode_attn_fp8
 * (kv_dtype PKV_KV_FP8) or paged_decode_attn_bf16 (PKV_KV_BF16) chooses for
 * these sizes and this num_ctas on the current device, without launching
 * anything: *cluster_size = 0 for split-K (a partial kernel and a merge
 * kernel), C > 0 for cluster mode (one kernel of clusters of C CTAs);
 * *ctas = CTAs of the partial kernel; *launches = kernels one call launches
 * (2 or 1).  The choice depends only on these arguments and the device, never
 * on the device-side lengths.  Returns PKV_ERR_INVALID_ARG /
 * PKV_ERR_UNSUPPORTED for arguments the attention call would reject.
 */
PKV_API pkv_status paged_decode_attn_plan(int32_t kv_dtype, int32_t batch, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          int32_t max_pages, int32_t page_size, int32_t num_ctas,
                                          int32_t* cluster_size, int32_t* ctas,
                                          int32_t* launches);

/*
 * paged_decode_attn_fp8 -- decode attention of one new query token per
 * request over a paged FP8 E4M3 cache, converting on every read ([T]
 * "量化 KV cache": the FP8 attention kernel converts values as it reads
 * them; [S] "KV 快取量化", Table 1).
 *
 * For every request b not aborted and every query head h (KV head
 * h / (num_q_heads / num_kv_heads)):
 *   s_t = sm_scale * sum_d q[b][h][d] * (decode(K_t[d]) * k_scale), t < L
 *   lse[b][h] = ln sum_t exp(s_t)        (natural log, scaled scores)
 *   out[b][h] = bf16( sum_t exp(s_t - lse[b][h]) * decode(V_t) * v_scale )
 * where token t of request b lives in page page_table[b][t / page_size],
 * slot t % page_size.  Aborted requests (abort[b] != 0), requests whose
 * length is outside [1, max_pages * page_size] and requests whose used
 * page-table entries name a page outside [0, num_pages) get out = 0 and
 * lse = -inf; the cache pages of an aborted request are never read into
 * the computation.
 *
 * q [batch][num_q_heads][head_dim] bf16 (16-byte aligned); caches as above
 * (16-byte aligned); out [batch][num_q_heads][head_dim] bf16; lse
 * [batch][num_q_heads] fp32.  workspace: device memory of at least
 * paged_decode_attn_workspace_size(PKV_KV_FP8, ...) bytes, 256-byte
 * aligned, not shared with a concurrently running attention call; its
 * contents need no initialisation.  Calls issued back to back on one stream
 * may share a workspace, with no synchronisation between them: apart from
 * clearing the status word (which no kernel reads), a call's kernels write
 * the workspace only after the previous kernel on the stream has finished.
 * num_ctas selects the work split (every choice gives the
 * same result up to rounding):
 *   0     the library chooses (cluster mode when the batch has no more
 *         (request, KV-head) items than the GPU holds resident CTAs, split-K
 *         over one wave otherwise);
 *   N > 0 split-K over N CTAs;
 *   -C    cluster mode with clusters of C CTAs, 1 <= C <= 16
 *         (PKV_ERR_UNSUPPORTED if the device cannot run that cluster size).
 *
 * Work split.  Split-K: the (request, KV head, 64-token chunk) units are
 * divided evenly over the CTAs of one persistent wave, and a request split
 * over several CTAs is combined by a log-sum-exp merge kernel (a second
 * launch).  Cluster mode: one launch of K thread-block clusters of C CTAs;
 * cluster k owns whole items, whose units its C CTAs divide evenly, and the
 * CTAs of a cluster combine the partial results of the items they share in
 * distributed shared memory; no merge kernel runs and the workspace is used
 * only for its status word.  Before its grid dependency wait the kernel
 * reads q, seq_lens and page_table and prefetches its first K/V tiles into
 * L2; everything else (abort, the cache contents) is read after the
 * preceding kernel on the stream has finished.
 */
PKV_API pkv_status paged_decode_attn_fp8(const uint16_t* q, const uint8_t* k_cache,
                                 const uint8_t* v_cache, float k_scale, float v_scale,
                                 const int32_t* page_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                                 int32_t num_pages, float sm_scale, const uint8_t* abort,
                                 uint16_t* out, float* lse, void* workspace,
                                 size_t workspace_bytes, int32_t num_ctas, void* stream);

/*
 * paged_decode_attn_fp8_prefix -- paged_decode_attn_fp8 for batches whose
 * requests share leading cache pages (a common prompt beginning whose pages
 * several requests' page tables name: [T] "保护共享 KV cache", where cache
 * reuse puts many requests on the same physical pages; [R], the prefix
 * caching remark in "为什么 Cloudflare 的小型缓存胜过单纯的速度").  Same
 * arguments, same outputs (up to rounding) and same abort / invalid-input
 * behaviour as paged_decode_attn_fp8; the shared pages are read once per
 * group instead of once per request.
 *
 * Nothing about the sharing is passed in: the call finds it on the device.
 * Request b joins request b - 1's group when their page tables name the same
 * valid pages for at least 4 leading 64-token chunks that lie entirely before
 * both requests' newest tokens (only consecutive requests form groups).  A
 * group's reference row is its member with the most chunks before its newest
 * token (the first on a tie); each member shares with the group the leading
 * chunks it has in common with the reference row (same rule).  Runs of up to
 * 64 / G consecutive members from the group's first request
 * (G = num_q_heads / num_kv_heads) form tensor-core tiles of two KV heads
 * when a run has at least 2 members and one of them other than the
 * reference shares at least 4 chunks; the tile covers the run's largest
 * share, which the reference, if in the run, takes as its own.  Those
 * chunks are attended for all members of the tile together; a member with
 * at most 2 chunks after them is finished in the tile too, the others'
 * remaining chunks go through the split-K kernel, and a merge kernel
 * combines the two.  Supported: head_dim 128, an even num_kv_heads and
 * G <= 8; other shapes run paged_decode_attn_fp8 unchanged (nothing
 * shared).
 *
 * workspace: at least paged_decode_attn_fp8_prefix_workspace_size(...)
 * bytes (the split-K workspace plus one partial record per (request, pair of
 * KV heads) and the group plan), 256-byte aligned, no initialisation needed;
 * word 0 is the status word as for paged_decode_attn_fp8.  num_ctas: 0 (the
 * library's split-K grid) or N > 0 (split-K over N CTAs); cluster mode is
 * not used (PKV_ERR_INVALID_ARG for num_ctas < 0).  chunk_begin_out: NULL,
 * or a device [batch] int32 array that receives, per request, the number of
 * leading chunks attended in its tile (0 = none; all of its chunks when the
 * tile finished it), in stream order.
 * Kernels: four plan kernels, the shared-prefix kernel, the split-K partial
 * kernel and the merge kernel, all chained with programmatic dependent
 * launch; none of them reads the cache, the page table or abort before the
 * preceding kernel has finished except the first, which reads seq_lens and
 * page_table (inputs no kernel writes).
 */
PKV_API size_t paged_decode_attn_fp8_prefix_workspace_size(int32_t batch, int32_t num_q_heads,
                                                           int32_t num_kv_heads,
                                                           int32_t head_dim, int32_t num_ctas);
PKV_API pkv_status paged_decode_attn_fp8_prefix(const uint16_t* q, const uint8_t* k_cache,
                                                const uint8_t* v_cache, float k_scale,
                                                float v_scale, const int32_t* page_table,
                                                int32_t max_pages, const int32_t* seq_lens,
                                                int32_t batch, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t page_size, int32_t num_pages,
                                                float sm_scale, const uint8_t* abort,
                                                uint16_t* out, float* lse, void* workspace,
                                                size_t workspace_bytes, int32_t num_ctas,
                                                int32_t* chunk_begin_out, void* stream);

/*
 * paged_decode_attn_bf16 -- the same attention over a BF16 cache (no
 * scales), the comparison kernel of [S] Table 1.  Workspace from
 * paged_decode_attn_workspace_size(PKV_KV_BF16, ...).
 */
PKV_API pkv_status paged_decode_attn_bf16(const uint16_t* q, const uint16_t* k_cache,
                                  const uint16_t* v_cache, const int32_t* page_table,
                                  int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t page_size, int32_t num_pages, float sm_scale,
                                  const uint8_t* abort, uint16_t* out, float* lse,
                                  void* workspace, size_t workspace_bytes, int32_t num_ctas,
                                  void* stream);

/*
 * paged_decode_attn_fp8_noalloc -- paged_decode_attn_fp8 for callers that
 * cannot allocate device memory.  The source pages have no counterpart to
 * this call; it exists for integration only.
 *
 * Some callers cannot hand the attention call a workspace: a plugin whose
 * host framework passes it only its inputs and outputs and owns every other
 * allocation, or a latency-critical path where cudaMalloc / cudaFree would
 * implicitly synchronise the device.  This call takes the same arguments as
 * paged_decode_attn_fp8 without the workspace and runs the same kernels,
 * using instead a scratch array compiled into the library:
 *   - its size is paged_decode_attn_fp8_noalloc_scratch_bytes() (8 MiB); every
 *     GPU that loads the library holds it until the process exits;
 *   - sizes whose workspace (paged_decode_attn_workspace_size(PKV_KV_FP8, ...))
 *     would exceed it are rejected with PKV_ERR_WORKSPACE and a message; with
 *     the default grid on a B200 that is roughly batch * num_kv_heads > 1700
 *     at head_dim 128 and a GQA group of 8;
 *   - the first call on a device looks up the array's device address for that
 *     device (make that first call before any stream capture);
 *   - the call allocates and frees nothing; the kernels write every scratch
 *     value before reading it (the array keeps the previous call's contents),
 *     including the status word, which paged_decode_attn_fp8_noalloc_status
 *     copies out;
 *   - all calls on a device share the one array, so two calls whose work
 *     overlaps on the GPU (different streams, or different host threads
 *     without ordering) race and corrupt each other's results.
 */
PKV_API pkv_status paged_decode_attn_fp8_noalloc(const uint16_t* q, const uint8_t* k_cache,
                                         const uint8_t* v_cache, float k_scale, float v_scale,
                                         const int32_t* page_table, int32_t max_pages,
                                         const int32_t* seq_lens, int32_t batch,
                                         int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t page_size, int32_t num_pages,
                                         float sm_scale, const uint8_t* abort, uint16_t* out,
                                         float* lse, int32_t num_ctas, void* stream);

/* Bytes of the built-in scratch used by paged_decode_attn_fp8_noalloc. */
PKV_API size_t paged_decode_attn_fp8_noalloc_scratch_bytes(void);

/*
 * paged_decode_attn_fp8_noalloc_status -- enqueues on `stream` a copy of the
 * current device's built-in scratch status word (4 bytes) to status_out,
 * host or device memory.  The word is the one paged_decode_attn_fp8 reports
 * in its workspace: 0, or 1 if an internal bounded wait expired in the last
 * no-allocation call on that device.  The copy is stream-ordered: issue it
 * after the call on the same stream and read status_out once the stream has
 * finished (a pageable host destination makes the copy synchronous).
 * Allocates nothing.  Returns PKV_ERR_INVALID_ARG if status_out is NULL.
 */
PKV_API pkv_status paged_decode_attn_fp8_noalloc_status(uint32_t* status_out, void* stream);

/*
 * int4_dequant_gemv -- y = x W^T with W stored as 4-bit integer codes and
 * expanded to floating point before the multiply, the decode-time use of
 * INT4 weights ([T] "压缩模型权重": decode streams every weight once per
 * token, so 4-bit codes cut the bytes per token; [S] "模型權重壓縮：GLM 5.2
 * 從 705 GB 縮到 421 GB", Table 2: FP8 vs INT4 decode throughput against
 * concurrency; [R] "GLM 权重压缩改变了阶段权衡").  The pages fix no format;
 * this call's:
 *   x       [batch][k] bf16 activations (16-byte aligned);
 *   w_tiles n * k / 2 bytes (16-byte aligned) of signed two's complement
 *           4-bit codes (-8..7) in tiles of 128 rows x 256 columns: tile
 *           (r, t), rows 128r.. and columns 256t.., is 16384 bytes at byte
 *           (r * (k/256) + t) * 16384; inside it row j's 128 bytes start at
 *           (j mod 128) * 128 and hold 32 little-endian 32-bit words, word w
 *           covering columns 256t + 8w .. +7: column 8w + 2i sits in bits
 *           4i .. 4i+3 and column 8w + 2i + 1 in bits 16 + 4i .. 19 + 4i
 *           (i = 0..3: the even columns in the low half-word, the odd ones
 *           in the high half-word; each tile is one contiguous read).
 *           int4_tile_layout in the Python binding re-lays a row-major
 *           matrix of codes into this format;
 *   scales  n * k / group_size bf16 (16-byte aligned): the scale of rows
 *           128r.. for columns g*group_size.. is the 128-value run starting
 *           at element (r * (k/group_size) + g) * 128, one value per row;
 *   y       [batch][n] bf16 (2-byte aligned), written as
 *           y[b][j] = bf16_rne( sum_i x[b][i] * code(j, i) * scale(j, i / group_size) )
 *           with fp32 accumulation (the codes are exact in bf16 and each
 *           group is summed before it is scaled).
 * Sizes: 1 <= batch <= 64, n a positive multiple of 128, k a positive
 * multiple of 256, group_size = 128; anything else returns
 * PKV_ERR_INVALID_ARG or PKV_ERR_UNSUPPORTED without launching.
 * status: nullable device word; the kernel sets bit 0 if an internal bounded
 * wait expires (never expected; y is then unspecified).  All buffers are the
 * caller's; the call allocates nothing and is asynchronous on `stream`.
 */
PKV_API pkv_status int4_dequant_gemv(const uint16_t* x, const uint8_t* w_tiles,
                                     const uint16_t* scales, int32_t batch, int32_t n,
                                     int32_t k, int32_t group_size, uint16_t* y,
                                     uint32_t* status, void* stream);

/* Message describing the last non-OK status returned on this thread. */
PKV_API const char* pkv_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
PKV_API int32_t pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
