// kv_write.cu -- the batched page-tag check, the FP8 / BF16 append of the
// new token, and the BF16 -> FP8 page handoff.
//
// Source pages: "大模型推理优化：量化、压缩与安全验证", sections "量化 KV cache"
// (FP8 e4m3 cache) and "保护共享 KV cache" (per-page tags, per-request
// expected tags, check before a decode op reads the cache, abort on
// mismatch, done as a separate batched check); siami.tw editorial, section
// "共享 KV 快取的完整性檢查" (Table 3 and the note that the check is not fused
// into the attention kernel).
#include "device.cuh"
#include "internal.h"

namespace pkv {

// ---------------------------------------------------------------------------
// tag check: one CTA per request; threads stride over its used entries
// ---------------------------------------------------------------------------
constexpr int kTagThreads = 128;

__global__ void __launch_bounds__(kTagThreads)
tag_check_kernel(const uint32_t* __restrict__ page_tags, int32_t num_pages,
                 const int32_t* __restrict__ page_table,
                 const uint32_t* __restrict__ expected_tags, int32_t max_pages,
                 const int32_t* __restrict__ seq_lens, int32_t page_size,
                 uint8_t* __restrict__ abort_out, int32_t* __restrict__ num_aborted) {
    // Let the next kernel on the stream launch at once (its own prologue
    // overlaps this grid); it still waits for this grid to finish before it
    // reads anything this grid writes.
    launch_dependents();
    grid_dependency_wait();
    const int b = blockIdx.x;
    const int32_t L = seq_lens[b];
    int bad = (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_pages) * page_size);
    if (!bad) {
        const int32_t used = (L + page_size - 1) / page_size;
        const int32_t* row = page_table + static_cast<int64_t>(b) * max_pages;
        const uint32_t* exp = expected_tags + static_cast<int64_t>(b) * max_pages;
#pragma unroll 4
        for (int j = threadIdx.x; j < used; j += kTagThreads) {
            const int32_t pid = row[j];
            const uint32_t want = exp[j];
            if (pid < 0 || pid >= num_pages)
                bad = 1;
            else if (__ldg(page_tags + pid) != want)
                bad = 1;
        }
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        abort_out[b] = static_cast<uint8_t>(bad != 0);
        if (bad && num_aborted) atomicAdd(num_aborted, 1);
    }
}

cudaError_t launch_tag_check(const uint32_t* page_tags, int32_t num_pages,
                             const int32_t* page_table, const uint32_t* expected_tags,
                             int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                             int32_t page_size, uint8_t* abort_out, int32_t* num_aborted,
                             cudaStream_t stream) {
    PdlLaunch l(dim3(batch), dim3(kTagThreads), 0, stream);
    return cudaLaunchKernelEx(&l.cfg, tag_check_kernel, page_tags, num_pages, page_table,
                              expected_tags, max_pages, seq_lens, page_size, abort_out,
                              num_aborted);
}

// ---------------------------------------------------------------------------
// E4M3 quantisation of bf16 values: y = x / scale as one correctly rounded
// binary32 division, then the hardware's round-to-nearest-even conversion
// with saturation to +-448; a NaN input becomes S.1111.111 with its sign.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t quantize_pair(float x_lo, float x_hi, float scale) {
    const float y_lo = __fdiv_rn(x_lo, scale);
    const float y_hi = __fdiv_rn(x_hi, scale);
    uint32_t p = f32x2_to_e4m3x2(y_hi, y_lo);
    // The quotient of a NaN is a NaN of unspecified sign; the code takes the
    // sign of the input (a finite, positive scale makes y NaN iff x is).
    if (isnan(x_lo)) p = (p & 0xFF00u) | (signbit(x_lo) ? 0xFFu : 0x7Fu);
    if (isnan(x_hi)) p = (p & 0x00FFu) | ((signbit(x_hi) ? 0xFFu : 0x7Fu) << 8);
    return p;
}
// 8 bf16 values (one 16-byte word) -> 8 codes (two 32-bit words).
__device__ __forceinline__ uint2 quantize8(uint4 raw, float scale) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        p[i] = quantize_pair(bf16_bits_to_f32(w[i] & 0xFFFFu), bf16_bits_to_f32(w[i] >> 16), scale);
    return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

// ---------------------------------------------------------------------------
// append: one CTA per request
// ---------------------------------------------------------------------------
constexpr int kAppendThreads = 256;

template <bool kFp8>
__global__ void __launch_bounds__(kAppendThreads)
append_kernel(const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
              const int32_t* __restrict__ page_table, int32_t max_pages,
              const int32_t* __restrict__ seq_lens, int32_t num_kv_heads, int32_t head_dim,
              int32_t page_size, float k_scale, float v_scale, void* __restrict__ k_cache,
              void* __restrict__ v_cache, int32_t num_pages, const uint8_t* __restrict__ abort) {
    // Let the next kernel on the stream launch at once (its own prologue
    // overlaps this grid); it still waits for this grid to finish before it
    // reads anything this grid writes.
    launch_dependents();
    grid_dependency_wait();
    const int b = blockIdx.x;
    const int32_t L = seq_lens[b];
    if (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_pages) * page_size) return;
    if (abort != nullptr && abort[b] != 0) return;
    const int32_t pos = L - 1;
    const int32_t pid = page_table[static_cast<int64_t>(b) * max_pages + pos / page_size];
    if (pid < 0 || pid >= num_pages) return;
    const int32_t slot = pos % page_size;
    const int per_tensor = num_kv_heads * (head_dim / 8);
    for (int e = threadIdx.x; e < 2 * per_tensor; e += kAppendThreads) {
        const bool is_v = e >= per_tensor;
        const int r = is_v ? e - per_tensor : e;
        const int h = r / (head_dim / 8);
        const int d8 = r % (head_dim / 8);
        const uint16_t* src = (is_v ? v_new : k_new) +
                              (static_cast<int64_t>(b) * num_kv_heads + h) * head_dim + d8 * 8;
        const uint4 raw = *reinterpret_cast<const uint4*>(src);
        const int64_t dst =
            ((static_cast<int64_t>(pid) * num_kv_heads + h) * page_size + slot) * head_dim + d8 * 8;
        if constexpr (kFp8) {
            uint8_t* cache = static_cast<uint8_t*>(is_v ? v_cache : k_cache);
            *reinterpret_cast<uint2*>(cache + dst) = quantize8(raw, is_v ? v_scale : k_scale);
        } else {
            uint16_t* cache = static_cast<uint16_t*>(is_v ? v_cache : k_cache);
            *reinterpret_cast<uint4*>(cache + dst) = raw;
        }
    }
}

cudaError_t launch_append(bool fp8, const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                          int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                          int32_t page_size, float k_scale, float v_scale, void* k_cache,
                          void* v_cache, int32_t num_pages, const uint8_t* abort,
                          cudaStream_t stream) {
    PdlLaunch l(dim3(batch), dim3(kAppendThreads), 0, stream);
    if (fp8)
        return cudaLaunchKernelEx(&l.cfg, append_kernel<true>, k_new, v_new, page_table,
                                  max_pages, seq_lens, num_kv_heads, head_dim, page_size, k_scale,
                                  v_scale, k_cache, v_cache, num_pages, abort);
    return cudaLaunchKernelEx(&l.cfg, append_kernel<false>, k_new, v_new, page_table, max_pages,
                              seq_lens, num_kv_heads, head_dim, page_size, k_scale, v_scale,
                              k_cache, v_cache, num_pages, abort);
}

// ---------------------------------------------------------------------------
// fused check + append: one CTA per request.  The request's tag check and its
// append depend on nothing but the request itself, so one CTA checks the used
// entries while the new token's K/V are already being loaded, and writes the
// token only if the request passed.  Results are those of kv_tag_check
// followed by kv_append_* with its abort mask.
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = 256;

template <bool kFp8>
__global__ void __launch_bounds__(kFusedThreads)
check_append_kernel(const uint32_t* __restrict__ page_tags, int32_t num_pages,
                    const int32_t* __restrict__ page_table,
                    const uint32_t* __restrict__ expected_tags, int32_t max_pages,
                    const int32_t* __restrict__ seq_lens, int32_t page_size,
                    const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                    int32_t num_kv_heads, int32_t head_dim, float k_scale, float v_scale,
                    void* __restrict__ k_cache, void* __restrict__ v_cache,
                    uint8_t* __restrict__ abort_out, int32_t* __restrict__ num_aborted) {
    launch_dependents();
    grid_dependency_wait();
    const int b = blockIdx.x;
    const int per_tensor = num_kv_heads * (head_dim / 8);
    const int32_t* row = page_table + static_cast<int64_t>(b) * max_pages;
    const uint32_t* exp = expected_tags + static_cast<int64_t>(b) * max_pages;
    // One round trip for everything that does not depend on the length: the
    // length itself, this thread's first page-table entry and expected tag,
    // and the new token's values for this thread's first two 8-element groups.
    const int32_t L = seq_lens[b];
    const int j0 = threadIdx.x;
    const int32_t p_first = j0 < max_pages ? row[j0] : -1;
    const uint32_t e_first = j0 < max_pages ? exp[j0] : 0u;
    uint4 raw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int e = threadIdx.x + k * kFusedThreads;
        if (e < 2 * per_tensor) {
            const bool is_v = e >= per_tensor;
            const int r = is_v ? e - per_tensor : e;
            const int h = r / (head_dim / 8), d8 = r % (head_dim / 8);
            raw[k] = *reinterpret_cast<const uint4*>(
                (is_v ? v_new : k_new) + (static_cast<int64_t>(b) * num_kv_heads + h) * head_dim +
                d8 * 8);
        }
    }
    int bad = (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_pages) * page_size);
    int32_t pid = -1, slot = 0;
    if (!bad) {
        const int32_t pos = L - 1;
        slot = pos % page_size;
        const int32_t used = (L + page_size - 1) / page_size;
        pid = row[pos / page_size];
        for (int j = j0; j < used; j += kFusedThreads) {
            const int32_t p = (j == j0) ? p_first : row[j];
            const uint32_t want = (j == j0) ? e_first : exp[j];
            if (p < 0 || p >= num_pages)
                bad = 1;
            else if (__ldg(page_tags + p) != want)
                bad = 1;
        }
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        abort_out[b] = static_cast<uint8_t>(bad != 0);
        if (bad && num_aborted) atomicAdd(num_aborted, 1);
    }
    if (bad) return;   // an aborted request writes nothing (its last page id was checked too)
    int k = 0;
    for (int e = threadIdx.x; e < 2 * per_tensor; e += kFusedThreads, ++k) {
        const bool is_v = e >= per_tensor;
        const int r = is_v ? e - per_tensor : e;
        const int h = r / (head_dim / 8), d8 = r % (head_dim / 8);
        uint4 val;
        if (k == 0)
            val = raw[0];
        else if (k == 1)
            val = raw[1];
        else
            val = *reinterpret_cast<const uint4*>(
                (is_v ? v_new : k_new) + (static_cast<int64_t>(b) * num_kv_heads + h) * head_dim +
                d8 * 8);
        const int64_t dst =
            ((static_cast<int64_t>(pid) * num_kv_heads + h) * page_size + slot) * head_dim + d8 * 8;
        if constexpr (kFp8) {
            uint8_t* cache = static_cast<uint8_t*>(is_v ? v_cache : k_cache);
            *reinterpret_cast<uint2*>(cache + dst) = quantize8(val, is_v ? v_scale : k_scale);
        } else {
            uint16_t* cache = static_cast<uint16_t*>(is_v ? v_cache : k_cache);
            *reinterpret_cast<uint4*>(cache + dst) = val;
        }
    }
}

cudaError_t launch_check_append(bool fp8, const uint32_t* page_tags, int32_t num_pages,
                                const int32_t* page_table, const uint32_t* expected_tags,
                                int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                int32_t page_size, const uint16_t* k_new, const uint16_t* v_new,
                                int32_t num_kv_heads, int32_t head_dim, float k_scale,
                                float v_scale, void* k_cache, void* v_cache, uint8_t* abort_out,
                                int32_t* num_aborted, cudaStream_t stream) {
    PdlLaunch l(dim3(batch), dim3(kFusedThreads), 0, stream);
    if (fp8)
        return cudaLaunchKernelEx(&l.cfg, check_append_kernel<true>, page_tags, num_pages,
                                  page_table, expected_tags, max_pages, seq_lens, page_size, k_new,
                                  v_new, num_kv_heads, head_dim, k_scale, v_scale, k_cache, v_cache,
                                  abort_out, num_aborted);
    return cudaLaunchKernelEx(&l.cfg, check_append_kernel<false>, page_tags, num_pages, page_table,
                              expected_tags, max_pages, seq_lens, page_size, k_new, v_new,
                              num_kv_heads, head_dim, k_scale, v_scale, k_cache, v_cache,
                              abort_out, num_aborted);
}

// ---------------------------------------------------------------------------
// page reallocation bookkeeping: tag bumps and expected-tag rebuilds
// ("保护共享 KV cache": a page's tag changes whenever it is reallocated; the
// server records each request's expected tags)
// ---------------------------------------------------------------------------
constexpr int kTagOpThreads = 256;

__global__ void __launch_bounds__(kTagOpThreads)
retag_kernel(uint32_t* __restrict__ page_tags, int32_t num_pages,
             const int32_t* __restrict__ pages, int32_t n) {
    launch_dependents();
    grid_dependency_wait();
    for (int i = blockIdx.x * kTagOpThreads + threadIdx.x; i < n; i += gridDim.x * kTagOpThreads) {
        const int32_t p = pages[i];
        if (p >= 0 && p < num_pages) atomicAdd(page_tags + p, 1u);   // wraps mod 2^32
    }
}

__global__ void __launch_bounds__(kTagOpThreads)
expected_tags_kernel(const uint32_t* __restrict__ page_tags, int32_t num_pages,
                     const int32_t* __restrict__ page_table, int32_t max_pages,
                     const int32_t* __restrict__ seq_lens, int32_t page_size,
                     uint32_t* __restrict__ expected_tags) {
    launch_dependents();
    grid_dependency_wait();
    const int b = blockIdx.x;
    const int32_t L = seq_lens[b];
    if (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_pages) * page_size) return;
    const int32_t used = (L + page_size - 1) / page_size;
    const int64_t row = static_cast<int64_t>(b) * max_pages;
    for (int j = threadIdx.x; j < used; j += kTagOpThreads) {
        const int32_t p = page_table[row + j];
        if (p >= 0 && p < num_pages) expected_tags[row + j] = page_tags[p];
    }
}

cudaError_t launch_retag(uint32_t* page_tags, int32_t num_pages, const int32_t* pages, int32_t n,
                         cudaStream_t stream) {
    int blocks = (n + kTagOpThreads - 1) / kTagOpThreads;
    if (blocks > 1024) blocks = 1024;
    PdlLaunch l(dim3(blocks), dim3(kTagOpThreads), 0, stream);
    return cudaLaunchKernelEx(&l.cfg, retag_kernel, page_tags, num_pages, pages, n);
}

cudaError_t launch_expected_tags(const uint32_t* page_tags, int32_t num_pages,
                                 const int32_t* page_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t batch, int32_t page_size,
                                 uint32_t* expected_tags, cudaStream_t stream) {
    PdlLaunch l(dim3(batch), dim3(kTagOpThreads), 0, stream);
    return cudaLaunchKernelEx(&l.cfg, expected_tags_kernel, page_tags, num_pages, page_table,
                              max_pages, seq_lens, page_size, expected_tags);
}

// ---------------------------------------------------------------------------
// BF16 -> FP8 page handoff: grid-stride over 16-element groups
// ---------------------------------------------------------------------------
constexpr int kRequantThreads = 256;

__global__ void __launch_bounds__(kRequantThreads)
requant_kernel(const uint16_t* __restrict__ src_pool, int32_t src_num_pages,
               const int32_t* __restrict__ src_pages, uint8_t* __restrict__ dst_pool,
               int32_t dst_num_pages, const int32_t* __restrict__ dst_pages, int32_t num_pairs,
               int64_t page_elems, float scale) {
    // Let the next kernel on the stream launch at once (its own prologue
    // overlaps this grid); it still waits for this grid to finish before it
    // reads anything this grid writes.
    launch_dependents();
    grid_dependency_wait();
    const int64_t groups = page_elems / 16;
    const int64_t total = static_cast<int64_t>(num_pairs) * groups;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t pair = static_cast<int32_t>(i / groups);
        const int64_t gi = i % groups;
        const int32_t s = src_pages[pair];
        const int32_t d = dst_pages[pair];
        if (s < 0 || s >= src_num_pages || d < 0 || d >= dst_num_pages) continue;
        const uint4* sp = reinterpret_cast<const uint4*>(src_pool + s * page_elems + gi * 16);
        const uint2 lo = quantize8(sp[0], scale);
        const uint2 hi = quantize8(sp[1], scale);
        *reinterpret_cast<uint4*>(dst_pool + d * page_elems + gi * 16) =
            make_uint4(lo.x, lo.y, hi.x, hi.y);
    }
}

cudaError_t launch_requant(const uint16_t* src_pool, int32_t src_num_pages,
                           const int32_t* src_pages, uint8_t* dst_pool, int32_t dst_num_pages,
                           const int32_t* dst_pages, int32_t num_pairs, int64_t page_elems,
                           float scale, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t total = static_cast<int64_t>(num_pairs) * (page_elems / 16);
    int64_t blocks = (total + kRequantThreads - 1) / kRequantThreads;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    PdlLaunch l(dim3(static_cast<unsigned>(blocks)), dim3(kRequantThreads), 0, stream);
    return cudaLaunchKernelEx(&l.cfg, requant_kernel, src_pool, src_num_pages, src_pages,
                              dst_pool, dst_num_pages, dst_pages, num_pairs, page_elems, scale);
}

// The step's first kernels run beside the attention grid that programmatic
// dependent launch starts early: an SM running one of them must already have
// its on-chip memory configured as the attention kernel wants it (all of it
// shared), or the attention CTAs can join that SM only after it drains.
cudaError_t step_kernels_set_carveout() {
    const int c = cudaSharedmemCarveoutMaxShared;
    const cudaFuncAttribute at = cudaFuncAttributePreferredSharedMemoryCarveout;
    cudaError_t e = cudaFuncSetAttribute(tag_check_kernel, at, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(append_kernel<true>, at, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(append_kernel<false>, at, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(check_append_kernel<true>, at, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(check_append_kernel<false>, at, c);
    return e;
}

}  // namespace pkv
