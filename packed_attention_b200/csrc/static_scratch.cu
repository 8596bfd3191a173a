// mf_joint_attn_fwd_static_scratch: the joint forward for callers that cannot
// allocate device memory (a plugin handed a stream but no allocator, code
// inside a global-mode stream capture where cudaMalloc is illegal, or a
// latency-critical loop that cannot pay for cudaMalloc's implicit device
// synchronisation). The scratch the forward needs (q_hat and k_hat) comes
// from a fixed array compiled into the library instead of from the caller.
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library
// call.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/mf_attn.h"

namespace {

constexpr size_t kScratchBytes = MF_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per GPU that loads the library, held until the process exits. In
// host code this name is only a stand-in for the symbol: the device address
// must come from cudaGetSymbolAddress (below), never from taking &g_scratch.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device, cached only once a lookup has
// succeeded: a failed lookup (for example one attempted while the stream is
// being captured) leaves the slot empty, and the next call tries again.
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Address of g_scratch on the current device (looked up with that device
// current), or NULL if the lookup failed; the failure's error state is
// cleared so that it does not surface at an unrelated later call.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return nullptr;
  }
  // Two threads may both look it up; they find the same address.
  g_scratch_ptr[dev].store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" mf_status mf_joint_attn_fwd_static_scratch(
    const void* q, const void* k, const void* v, const float* g_q_text, const float* g_q_img,
    const float* g_k_text, const float* g_k_img, const int32_t* cu_seqlens_dev,
    const mf_segment* segs_dev, int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
    int32_t total_tokens, int32_t heads, int32_t head_dim, float eps, float softmax_scale,
    void* out, void* stream) {
  // Size first: a pack that does not fit is refused before anything runs.
  // (Invalid sizes give 0 here and are reported by mf_joint_attn_fwd.)
  if (mf_joint_attn_workspace_bytes(total_tokens, heads, head_dim) > kScratchBytes)
    return MF_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return MF_ERR_CUDA;
  // The prologue overwrites q_hat and k_hat on every call before the
  // attention kernel reads them, so whatever an earlier call left in the
  // array is never read.
  return mf_joint_attn_fwd(q, k, v, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev,
                           segs_dev, n_samples, work_dev, n_work, total_tokens, heads, head_dim,
                           eps, softmax_scale, out, scratch, kScratchBytes, stream);
}
