// paged_decode_attention_noalloc: the split-KV decode without a caller
// workspace. The split partials (m, l, u) live in a fixed-size array in the
// library's own device memory instead of a buffer the caller allocates.
//
// Why it exists: some callers cannot call cudaMalloc (or any allocator) at
// the point where they run decode -- e.g. a plug-in hosted by an inference
// server that owns every device allocation and hands the plug-in only its
// input and output tensors, or code on a latency-critical path that is not
// allowed to allocate at all. Those callers still pass q, the K/V pools,
// block tables, lengths and the output; the scratch below replaces the
// workspace argument.
//
// Cost and limits:
//   * every GPU that loads this library holds kScratchBytes of device memory
//     for the array until the process exits;
//   * the first call on a device looks up the array's device address with
//     cudaGetSymbolAddress (which may load the module); make that first call
//     before any stream capture on that device;
//   * all calls share the one array: two calls whose kernels overlap on the
//     GPU (different streams without ordering) race on it. Calls on one
//     stream are ordered and safe. Nothing in it needs to start at zero (each
//     split writes its partial before the combine kernel reads it);
//   * the array's device address is looked up once per device and kept for
//     the life of the process; it does not survive cudaDeviceReset of that
//     device (a process that resets a device must not call this entry point
//     on it afterwards);
//   * with num_splits == 0, when the automatic choice's partials would not
//     fit, the largest explicit split count whose partials fit is used
//     instead (down to 1, which needs no scratch); an explicit num_splits
//     whose partials would not fit returns KV_ERR_WORKSPACE.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "kvpaged.h"

namespace {

constexpr size_t kScratchBytes = KV_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_split_scratch on the current device (host code cannot
// use the symbol itself: in host code it names a host-side stand-in).
int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KV_ERR_CUDA;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_split_scratch) != cudaSuccess || !p) return KV_ERR_CUDA;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return KV_OK;
}

}  // namespace

extern "C" int paged_decode_attention_noalloc(float* out, const void* q, const void* k_pages, const void* v_pages,
                                              const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens,
                                              int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size,
                                              int32_t num_pages, float scale, int32_t dtype, int32_t num_splits,
                                              int* err_flag, void* stream) {
    if (B < 0 || H_q <= 0 || H_kv <= 0 || Dh <= 0 || max_blocks <= 0 || page_size <= 0 || num_splits < 0)
        return KV_ERR_ARG;
    size_t need = 0;
    int rc = paged_decode_workspace_bytes(B, H_q, H_kv, Dh, max_blocks, page_size, num_splits, &need);
    if (rc != KV_OK) return rc;
    if (need > kScratchBytes && num_splits == 0) {
        // automatic choice too large for the array: the largest explicit split count that fits
        int32_t s0 = 0;
        rc = paged_decode_num_splits(B, H_kv, max_blocks, page_size, 0, &s0);
        if (rc != KV_OK) return rc;
        for (int32_t s = s0 > 1 ? s0 - 1 : 8; s >= 1; --s) {
            rc = paged_decode_workspace_bytes(B, H_q, H_kv, Dh, max_blocks, page_size, s, &need);
            if (rc != KV_OK) return rc;
            if (need <= kScratchBytes) {
                num_splits = s;
                break;
            }
        }
    }
    if (need > kScratchBytes) return KV_ERR_WORKSPACE;  // partials exceed the fixed scratch
    void* scratch = nullptr;
    if (need > 0) {
        rc = scratch_for_current_device(&scratch);
        if (rc != KV_OK) return rc;
    }
    return paged_decode_attention(out, q, k_pages, v_pages, block_tables, max_blocks, seq_lens, B, H_q, H_kv, Dh,
                                  page_size, num_pages, scale, dtype, num_splits, scratch, need ? kScratchBytes : 0,
                                  err_flag, stream);
}
