// varlen_attn_noalloc.cu -- pqk_varlen_attn_fwd_noalloc: the packed varlen
// attention for callers that cannot allocate device memory.
//
// pqk_varlen_attn_fwd needs a small device workspace for its tile schedule,
// which the caller allocates and passes in. Some callers cannot do that: a
// plugin or an embedded runtime that is handed only its input and output
// buffers, under a host framework that owns the whole device heap through
// its own pool and offers no way to obtain an extra buffer. For them this
// entry point keeps the schedule in a fixed array in the library's own
// device memory (a file-scope __device__ array, present on every GPU that
// loads the library until the process exits), so the caller passes only
// inputs and outputs.
//
// Limits and sharing: the array holds the schedule of at most
// kNoAllocMaxRequests requests; larger B is rejected. Every call uses the
// same array and leaves its own schedule in it; the schedule kernel rewrites
// every word the attention kernel reads before it reads it, and resets the
// one word that must start at zero (the counter the attention's blocks claim
// work tiles with), so the previous call's contents never matter. Two calls whose work overlaps on the GPU (for example on
// two streams) race on the array and may produce wrong output: serialise
// them.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "pqk.h"
#include "pqk_internal.h"

namespace {

constexpr int kNoAllocMaxRequests = 4096;
// words of the schedule for kNoAllocMaxRequests requests (3B + 5: a header
// of 4 words, B + 1 tile offsets, 2B request words), rounded up to 256 bytes
// like the workspace size query
constexpr size_t kScratchWords = ((3 * static_cast<size_t>(kNoAllocMaxRequests) + 5) * 4 + 255) / 256 * 64;

static __device__ __align__(256) int32_t g_noalloc_schedule[kScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device, resolved once per
// device (the host-side symbol is only a stand-in, not a device address).
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_schedule) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int pqk_varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                           int64_t q_stride_t, int64_t k_stride_t, int64_t v_stride_t,
                                           int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T, int H,
                                           int D, float softmax_scale, void* stream) {
  if (B > kNoAllocMaxRequests) return PQK_ERR_WORKSPACE;
  if (B < 1) return PQK_ERR_INVALID_ARG;
  const size_t need = pqk_varlen_attn_workspace_size(B);
  if (need > sizeof(g_noalloc_schedule)) return PQK_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return PQK_ERR_CUDA;
  return pqk_varlen_attn_fwd(q, k, v, o, lse, q_stride_t, k_stride_t, v_stride_t, o_stride_t, cu_seqlens, B, T, H,
                             D, softmax_scale, scratch, sizeof(g_noalloc_schedule), stream);
}
