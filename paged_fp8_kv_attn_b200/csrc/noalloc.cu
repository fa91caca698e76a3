// noalloc.cu -- paged_decode_attn_fp8_noalloc: the FP8 decode-attention call
// for callers that cannot allocate device memory.
//
// The regular call takes its split-K scratch (status word, per-request chunk
// offsets and the partial results of requests split over several CTAs) as a
// caller-provided workspace.  Some callers have no way to provide one: for
// example a plugin whose host framework hands it only its inputs and outputs
// and owns every other allocation, or a latency-critical path where
// cudaMalloc / cudaFree would implicitly synchronise the device.  This entry
// point instead uses a fixed scratch array compiled into the library
// (kNoAllocScratchBytes of device memory that every GPU which loads the
// library holds until the process exits) and otherwise runs exactly the
// same kernels as paged_decode_attn_fp8.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "internal.h"
#include "pagedkv.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB

// In host code this name is only a stand-in for the symbol, not a device
// address: the address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the
// scratch array.
pkv_status scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        pkv::set_last_error("paged_decode_attn_fp8_noalloc: cudaGetDevice failed");
        return PKV_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        pkv::set_last_error("paged_decode_attn_fp8_noalloc: device index out of range");
        return PKV_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            char buf[256];
            snprintf(buf, sizeof buf,
                     "paged_decode_attn_fp8_noalloc: cudaGetSymbolAddress failed: %s",
                     cudaGetErrorString(e));
            pkv::set_last_error(buf);
            return PKV_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" PKV_API size_t paged_decode_attn_fp8_noalloc_scratch_bytes(void) {
    return kNoAllocScratchBytes;
}

extern "C" PKV_API pkv_status paged_decode_attn_fp8_noalloc(
    const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache, float k_scale,
    float v_scale, const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t page_size, int32_t num_pages, float sm_scale, const uint8_t* abort, uint16_t* out,
    float* lse, int32_t num_ctas, void* stream) {
    if (batch == 0) return PKV_OK;
    const size_t need = paged_decode_attn_workspace_size(PKV_KV_FP8, batch, num_q_heads,
                                                         num_kv_heads, head_dim, num_ctas);
    if (need == 0) return PKV_ERR_INVALID_ARG;   // message set by the size query
    if (need > kNoAllocScratchBytes) {
        char buf[320];
        snprintf(buf, sizeof buf,
                 "paged_decode_attn_fp8_noalloc: these sizes need %zu bytes of scratch but the "
                 "built-in scratch holds %zu bytes; pass a workspace to paged_decode_attn_fp8 "
                 "instead (or lower batch / num_ctas)",
                 need, kNoAllocScratchBytes);
        pkv::set_last_error(buf);
        return PKV_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    pkv_status st = scratch_for_current_device(&scratch);
    if (st != PKV_OK) return st;
    // The array keeps the previous call's contents; the kernels write every
    // word they read, the status word included, before reading it.
    return paged_decode_attn_fp8(q, k_cache, v_cache, k_scale, v_scale, page_table, max_pages,
                                 seq_lens, batch, num_q_heads, num_kv_heads, head_dim, page_size,
                                 num_pages, sm_scale, abort, out, lse, scratch,
                                 kNoAllocScratchBytes, num_ctas, stream);
}

extern "C" PKV_API pkv_status paged_decode_attn_fp8_noalloc_status(uint32_t* status_out,
                                                                  void* stream) {
    if (status_out == nullptr) {
        pkv::set_last_error("paged_decode_attn_fp8_noalloc_status: status_out is NULL");
        return PKV_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    pkv_status st = scratch_for_current_device(&scratch);
    if (st != PKV_OK) return st;
    // word 0 of the scratch is the status word of the attention workspace
    cudaError_t e = cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDefault,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        char buf[256];
        snprintf(buf, sizeof buf, "paged_decode_attn_fp8_noalloc_status: cudaMemcpyAsync: %s",
                 cudaGetErrorString(e));
        pkv::set_last_error(buf);
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}
