// C-ABI entry points of libmfattn: argument checks, workspace layout, TMA
// descriptor encoding and kernel launches on the caller's stream. All device
// code of the library lives in this translation unit (the kernels are in the
// included headers).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "../../include/mf_attn.h"
#include "attention_bwd.cuh"
#include "block.cuh"
#include "packed_attention.cuh"
#include "qk_prologue.cuh"
#include "qk_prologue_bwd.cuh"

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WorkspaceLayout {
  size_t q_hat;
  size_t k_hat;
  size_t total;
};

bool layout(int32_t total_tokens, int32_t heads, int32_t head_dim, WorkspaceLayout* w) {
  if (total_tokens < 1 || heads < 1 || (head_dim != 64 && head_dim != 128)) return false;
  const size_t tensor = round_up(static_cast<size_t>(total_tokens) * heads * head_dim * 2, kAlign);
  w->q_hat = 0;
  w->k_hat = tensor;
  w->total = 2 * tensor;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [T, H, d] bf16 viewed as a 3-D tensor (d, H, T); boxes of 64 dims x 1 head
// x 128 tokens with the 128-byte swizzle the MMA descriptors expect. Boxes
// that run past T are zero-filled.
bool encode_thd(CUtensorMap* map, const void* base, int32_t T, int32_t H, int32_t D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(mf::kSubM)};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows, cols] as a 2-D tensor (cols, rows) with
// boxes of 64 columns x box_rows rows and the 128-byte swizzle.
bool encode_matrix(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                   uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static std::once_flag once[kMaxDevices];
  static int count[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::call_once(once[dev], [dev] {
    int c = 0;
    count[dev] = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? c : 0;
  });
  return count[dev];
}

template <int D>
bool prepare_attention_kernel() {
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(once[dev], [dev] {
    // The kernel re-splits its registers between warpgroups; that only works
    // if it is launched with at least kMinLaunchRegs per thread (otherwise the
    // softmax warpgroups would wait forever for registers): refuse instead.
    cudaFuncAttributes attr;
    ok[dev] = cudaFuncGetAttributes(&attr, mf::packed_attention_kernel<D>) == cudaSuccess &&
              attr.numRegs >= mf::kMinLaunchRegs &&
              cudaFuncSetAttribute(mf::packed_attention_kernel<D>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mf::AttnConfig<D>::kSmemBytes) == cudaSuccess;
  });
  return ok[dev];
}

// Dynamic shared memory of the two backward attention kernels, set once per device.
template <int D>
bool prepare_bwd_kernels() {
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(once[dev], [dev] {
    ok[dev] = cudaFuncSetAttribute(mf::attn_bwd_dkdv_kernel<D>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mf::BwdConfig<D, false>::kSmemBytes) == cudaSuccess &&
              cudaFuncSetAttribute(mf::attn_bwd_dq_kernel<D>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mf::BwdConfig<D, true>::kSmemBytes) == cudaSuccess;
  });
  return ok[dev];
}

// Backward workspace: the forward's (q_hat, k_hat), then
// D [H, T] fp32, dq_hat and dk_hat [T, H, d] fp32 and the per-block partial
// gamma gradients [blocks, 4, d] fp32.
struct BwdLayout {
  WorkspaceLayout fwd;
  size_t delta, dq_hat, dk_hat, partial, total;
  int pro_blocks;
};

bool bwd_layout(int32_t total_tokens, int32_t heads, int32_t head_dim, BwdLayout* b) {
  if (!layout(total_tokens, heads, head_dim, &b->fwd)) return false;
  const size_t rows = static_cast<size_t>(total_tokens) * heads;
  const int tok_per_block = mf::kPrologueThreads / (head_dim / 8);
  b->pro_blocks = (total_tokens + tok_per_block - 1) / tok_per_block;
  b->delta = round_up(b->fwd.total, kAlign);
  b->dq_hat = b->delta + round_up(rows * 4, kAlign);
  b->dk_hat = b->dq_hat + round_up(rows * head_dim * 4, kAlign);
  b->partial = b->dk_hat + round_up(rows * head_dim * 4, kAlign);
  b->total = b->partial + round_up(static_cast<size_t>(b->pro_blocks) * 4 * head_dim * 4, kAlign);
  return true;
}

}  // namespace

extern "C" size_t mf_joint_attn_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim) {
  WorkspaceLayout w;
  return layout(total_tokens, heads, head_dim, &w) ? w.total : 0;
}

extern "C" mf_status mf_qk_prologue_3d(const void* q, const void* k, const float* g_q_text,
                                       const float* g_q_img, const float* g_k_text,
                                       const float* g_k_img, const int32_t* cu_seqlens_dev,
                                       const mf_segment* segs_dev, int32_t n_samples,
                                       int32_t total_tokens, int32_t heads, int32_t head_dim,
                                       float eps, int32_t frame_dims, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  WorkspaceLayout w;
  if (!layout(total_tokens, heads, head_dim, &w) || n_samples < 1 || !(eps >= 0.0f) ||
      !std::isfinite(eps))
    return MF_ERR_INVALID_ARG;
  if (frame_dims < 0 || frame_dims % 4 != 0 || frame_dims > head_dim - 4) return MF_ERR_INVALID_ARG;
  if (!q || !k || !g_q_text || !g_q_img || !g_k_text || !g_k_img || !cu_seqlens_dev || !segs_dev ||
      !workspace)
    return MF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MF_ERR_ALIGNMENT;
  if (workspace_bytes < w.total) return MF_ERR_WORKSPACE;
  const size_t bytes = static_cast<size_t>(total_tokens) * heads * head_dim * 2;
  if (overlaps(workspace, w.total, q, bytes) || overlaps(workspace, w.total, k, bytes))
    return MF_ERR_INVALID_ARG;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int tok_per_block = mf::kPrologueTokPerBlock;
  const unsigned grid = static_cast<unsigned>((total_tokens + tok_per_block - 1) / tok_per_block);
  if (head_dim == 128) {
    mf::qk_prologue_kernel<128><<<grid, mf::kPrologueThreads, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), g_q_text, g_q_img, g_k_text,
        g_k_img, cu_seqlens_dev, segs_dev, n_samples, total_tokens, heads, eps, frame_dims,
        reinterpret_cast<uint4*>(ws + w.q_hat), reinterpret_cast<uint4*>(ws + w.k_hat));
  } else {
    mf::qk_prologue_kernel<64><<<grid, mf::kPrologueThreads, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), g_q_text, g_q_img, g_k_text,
        g_k_img, cu_seqlens_dev, segs_dev, n_samples, total_tokens, heads, eps, frame_dims,
        reinterpret_cast<uint4*>(ws + w.q_hat), reinterpret_cast<uint4*>(ws + w.k_hat));
  }
  return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
}

extern "C" mf_status mf_qk_prologue(const void* q, const void* k, const float* g_q_text,
                                    const float* g_q_img, const float* g_k_text,
                                    const float* g_k_img, const int32_t* cu_seqlens_dev,
                                    const mf_segment* segs_dev, int32_t n_samples,
                                    int32_t total_tokens, int32_t heads, int32_t head_dim,
                                    float eps, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return mf_qk_prologue_3d(q, k, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev, segs_dev,
                           n_samples, total_tokens, heads, head_dim, eps, 0, workspace,
                           workspace_bytes, stream);
}

namespace {

// Stage 2 with an optional per-row log-normaliser output (lse, [heads, T]).
mf_status packed_attention_impl(const void* v, const mf_segment* segs_dev, int32_t n_samples,
                                const mf_work_item* work_dev, int32_t n_work,
                                int32_t total_tokens, int32_t heads, int32_t head_dim,
                                float softmax_scale, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  WorkspaceLayout w;
  if (!layout(total_tokens, heads, head_dim, &w) || n_samples < 1 || n_work < 1)
    return MF_ERR_INVALID_ARG;
  if (!v || !segs_dev || !work_dev || !out || !workspace) return MF_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MF_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MF_ERR_ALIGNMENT;
  if (workspace_bytes < w.total) return MF_ERR_WORKSPACE;
  const size_t bytes = static_cast<size_t>(total_tokens) * heads * head_dim * 2;
  if (overlaps(out, bytes, v, bytes) || overlaps(out, bytes, workspace, w.total))
    return MF_ERR_INVALID_ARG;
  if (lse) {
    const size_t lse_bytes = static_cast<size_t>(total_tokens) * heads * 4;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return MF_ERR_ALIGNMENT;
    if (overlaps(lse, lse_bytes, out, bytes) || overlaps(lse, lse_bytes, v, bytes) ||
        overlaps(lse, lse_bytes, workspace, w.total))
      return MF_ERR_INVALID_ARG;
  }

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUtensorMap tq, tk, tv;
  if (!encode_thd(&tq, ws + w.q_hat, total_tokens, heads, head_dim) ||
      !encode_thd(&tk, ws + w.k_hat, total_tokens, heads, head_dim) ||
      !encode_thd(&tv, v, total_tokens, heads, head_dim))
    return MF_ERR_CUDA;

  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  mf::AttnParams prm;
  prm.segs = segs_dev;
  prm.work = work_dev;
  prm.n_segs = n_samples;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.n_work = n_work;
  prm.heads = heads;
  prm.total_tokens = total_tokens;
  prm.scale_log2 = scale * 1.4426950408889634f;

  // Persistent: one CTA per SM (or fewer if there are fewer items).
  const int sms = sm_count();
  if (sms <= 0) return MF_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(n_work < sms ? n_work : sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 128) {
    if (!prepare_attention_kernel<128>()) return MF_ERR_CUDA;
    mf::packed_attention_kernel<128>
        <<<grid, mf::kAttnThreads, mf::AttnConfig<128>::kSmemBytes, s>>>(tq, tk, tv, prm);
  } else {
    if (!prepare_attention_kernel<64>()) return MF_ERR_CUDA;
    mf::packed_attention_kernel<64>
        <<<grid, mf::kAttnThreads, mf::AttnConfig<64>::kSmemBytes, s>>>(tq, tk, tv, prm);
  }
  return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
}

}  // namespace

extern "C" mf_status mf_packed_attention(const void* v, const mf_segment* segs_dev,
                                         int32_t n_samples, const mf_work_item* work_dev,
                                         int32_t n_work, int32_t total_tokens, int32_t heads,
                                         int32_t head_dim, float softmax_scale, void* out,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  return packed_attention_impl(v, segs_dev, n_samples, work_dev, n_work, total_tokens, heads,
                               head_dim, softmax_scale, out, nullptr, workspace, workspace_bytes,
                               stream);
}

extern "C" mf_status mf_joint_attn_fwd_3d(const void* q, const void* k, const void* v,
                                          const float* g_q_text, const float* g_q_img,
                                          const float* g_k_text, const float* g_k_img,
                                          const int32_t* cu_seqlens_dev,
                                          const mf_segment* segs_dev, int32_t n_samples,
                                          const mf_work_item* work_dev, int32_t n_work,
                                          int32_t total_tokens, int32_t heads, int32_t head_dim,
                                          float eps, int32_t frame_dims, float softmax_scale,
                                          void* out, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  // Check everything the second stage needs before launching the first.
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  if (!v || !work_dev || !out || n_work < 1 || !std::isfinite(softmax_scale))
    return MF_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(out)) return MF_ERR_ALIGNMENT;
  const size_t bytes = static_cast<size_t>(total_tokens > 0 ? total_tokens : 0) * heads * head_dim * 2;
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes)) return MF_ERR_INVALID_ARG;
  mf_status st = mf_qk_prologue_3d(q, k, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev,
                                   segs_dev, n_samples, total_tokens, heads, head_dim, eps,
                                   frame_dims, workspace, workspace_bytes, stream);
  if (st != MF_OK) return st;
  return mf_packed_attention(v, segs_dev, n_samples, work_dev, n_work, total_tokens, heads,
                             head_dim, softmax_scale, out, workspace, workspace_bytes, stream);
}

extern "C" mf_status mf_joint_attn_fwd(const void* q, const void* k, const void* v,
                                       const float* g_q_text, const float* g_q_img,
                                       const float* g_k_text, const float* g_k_img,
                                       const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                                       int32_t n_samples, const mf_work_item* work_dev,
                                       int32_t n_work, int32_t total_tokens, int32_t heads,
                                       int32_t head_dim, float eps, float softmax_scale, void* out,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  return mf_joint_attn_fwd_3d(q, k, v, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev,
                              segs_dev, n_samples, work_dev, n_work, total_tokens, heads, head_dim,
                              eps, 0, softmax_scale, out, workspace, workspace_bytes, stream);
}

namespace {

// y = 2^x through the same instruction the softmax uses for its exponentials.
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = mf::ex2_approx(x[i]);
}

}  // namespace

extern "C" mf_status mf_selftest_exp2(const float* x, float* y, int32_t n, void* stream) {
  if (!x || !y || n < 0) return MF_ERR_INVALID_ARG;
  if (n == 0) return MF_OK;
  selftest_exp2_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
}

namespace {

// One thread waits on an mbarrier that expects one arrival which never comes.
__global__ void selftest_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x != 0) return;
  mf::mbar_init(&bar, 1);
  abort_flag = 0;
  mf::fence_mbarrier_init();
  mf::wait_slow(&bar, 0, &abort_flag, limit_ns);  // records MF_ERR_TIMEOUT when it gives up
}

}  // namespace

extern "C" mf_status mf_selftest_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000) return MF_ERR_INVALID_ARG;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
}

extern "C" mf_status mf_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MF_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, mf::g_device_error, sizeof v) != cudaSuccess) return MF_ERR_CUDA;
  if (v != 0) {
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(mf::g_device_error, &zero, sizeof zero) != cudaSuccess)
      return MF_ERR_CUDA;
  }
  return static_cast<mf_status>(v);
}

extern "C" size_t mf_bwd_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim) {
  BwdLayout b;
  return bwd_layout(total_tokens, heads, head_dim, &b) ? b.total : 0;
}

extern "C" mf_status mf_joint_attn_fwd_lse(const void* q, const void* k, const void* v,
                                           const float* g_q_text, const float* g_q_img,
                                           const float* g_k_text, const float* g_k_img,
                                           const int32_t* cu_seqlens_dev,
                                           const mf_segment* segs_dev, int32_t n_samples,
                                           const mf_work_item* work_dev, int32_t n_work,
                                           int32_t total_tokens, int32_t heads, int32_t head_dim,
                                           float eps, int32_t frame_dims, float softmax_scale,
                                           void* out, float* lse, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  if (!v || !work_dev || !out || !lse || n_work < 1 || !std::isfinite(softmax_scale))
    return MF_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(out)) return MF_ERR_ALIGNMENT;
  const size_t bytes = static_cast<size_t>(total_tokens > 0 ? total_tokens : 0) * heads * head_dim * 2;
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes)) return MF_ERR_INVALID_ARG;
  const size_t lse_bytes = static_cast<size_t>(total_tokens > 0 ? total_tokens : 0) * heads * 4;
  if (overlaps(lse, lse_bytes, q, bytes) || overlaps(lse, lse_bytes, k, bytes))
    return MF_ERR_INVALID_ARG;
  mf_status st = mf_qk_prologue_3d(q, k, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev,
                                   segs_dev, n_samples, total_tokens, heads, head_dim, eps,
                                   frame_dims, workspace, workspace_bytes, stream);
  if (st != MF_OK) return st;
  return packed_attention_impl(v, segs_dev, n_samples, work_dev, n_work, total_tokens, heads,
                               head_dim, softmax_scale, out, lse, workspace, workspace_bytes,
                               stream);
}

extern "C" mf_status mf_joint_attn_bwd(
    const void* q, const void* k, const void* v, const float* g_q_text, const float* g_q_img,
    const float* g_k_text, const float* g_k_img, const void* out, const void* dout,
    const float* lse, const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
    int32_t n_samples, const mf_work_item* work_dev, int32_t n_work, int32_t total_tokens,
    int32_t heads, int32_t head_dim, float eps, int32_t frame_dims, float softmax_scale, void* dq,
    void* dk, void* dv, float* dgamma, void* workspace, size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  BwdLayout bl;
  if (!bwd_layout(total_tokens, heads, head_dim, &bl) || n_samples < 1 || n_work < 1)
    return MF_ERR_INVALID_ARG;
  if (!q || !k || !v || !g_q_text || !g_q_img || !g_k_text || !g_k_img || !out || !dout || !lse ||
      !cu_seqlens_dev || !segs_dev || !work_dev || !dq || !dk || !dv || !dgamma || !workspace)
    return MF_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps) || !std::isfinite(softmax_scale))
    return MF_ERR_INVALID_ARG;
  if (frame_dims < 0 || frame_dims % 4 != 0 || frame_dims > head_dim - 4) return MF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 || (reinterpret_cast<uintptr_t>(dgamma) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MF_ERR_ALIGNMENT;
  if (workspace_bytes < bl.total) return MF_ERR_WORKSPACE;
  const size_t bytes = static_cast<size_t>(total_tokens) * heads * head_dim * 2;
  const size_t lse_bytes = static_cast<size_t>(total_tokens) * heads * 4;
  const size_t g_bytes = static_cast<size_t>(4) * head_dim * 4;
  // Outputs must not overlap any input, the workspace or one another.
  struct Span { const void* p; size_t n; };
  const Span outs[4] = {{dq, bytes}, {dk, bytes}, {dv, bytes}, {dgamma, g_bytes}};
  const Span ins[7] = {{q, bytes}, {k, bytes}, {v, bytes}, {out, bytes}, {dout, bytes},
                       {lse, lse_bytes}, {workspace, bl.total}};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 7; ++j)
      if (overlaps(outs[i].p, outs[i].n, ins[j].p, ins[j].n)) return MF_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return MF_ERR_INVALID_ARG;
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // 1. q_hat, k_hat again (the forward's workspace need not have survived).
  mf_status st = mf_qk_prologue_3d(q, k, g_q_text, g_q_img, g_k_text, g_k_img, cu_seqlens_dev,
                                   segs_dev, n_samples, total_tokens, heads, head_dim, eps,
                                   frame_dims, workspace, workspace_bytes, stream);
  if (st != MF_OK) return st;
  const unsigned pro_grid = static_cast<unsigned>(bl.pro_blocks);
  float* delta = reinterpret_cast<float*>(ws + bl.delta);
  float* dq_hat = reinterpret_cast<float*>(ws + bl.dq_hat);
  float* dk_hat = reinterpret_cast<float*>(ws + bl.dk_hat);
  float* partial = reinterpret_cast<float*>(ws + bl.partial);

  CUtensorMap tq, tk, tv, tdo;
  if (!encode_thd(&tq, ws + bl.fwd.q_hat, total_tokens, heads, head_dim) ||
      !encode_thd(&tk, ws + bl.fwd.k_hat, total_tokens, heads, head_dim) ||
      !encode_thd(&tv, v, total_tokens, heads, head_dim) ||
      !encode_thd(&tdo, dout, total_tokens, heads, head_dim))
    return MF_ERR_CUDA;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  mf::BwdParams prm;
  prm.segs = segs_dev;
  prm.work = work_dev;
  prm.n_segs = n_samples;
  prm.lse = lse;
  prm.delta = delta;
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.q_rows = reinterpret_cast<const uint4*>(ws + bl.fwd.q_hat);
  prm.do_rows = static_cast<const uint4*>(dout);
  prm.n_work = n_work;
  prm.heads = heads;
  prm.total_tokens = total_tokens;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  const int sms = sm_count();
  if (sms <= 0) return MF_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(n_work < sms ? n_work : sms);

  auto run = [&](auto dtag) -> mf_status {
    constexpr int D = decltype(dtag)::value;
    if (!prepare_bwd_kernels<D>()) return MF_ERR_CUDA;
    // 2. D = rowsum(dO * out)
    mf::bwd_delta_kernel<D><<<pro_grid, mf::kPrologueThreads, 0, s>>>(
        static_cast<const uint4*>(out), static_cast<const uint4*>(dout), total_tokens, heads, delta);
    // 3. dv and dk_hat
    mf::BwdParams p1 = prm;
    p1.dhat = dk_hat;
    mf::attn_bwd_dkdv_kernel<D><<<grid, mf::kBwdThreads, mf::BwdConfig<D, false>::kSmemBytes, s>>>(
        tq, tk, tv, tdo, p1);
    // 4. dq_hat
    mf::BwdParams p2 = prm;
    p2.dhat = dq_hat;
    mf::attn_bwd_dq_kernel<D><<<grid, mf::kBwdThreads, mf::BwdConfig<D, true>::kSmemBytes, s>>>(
        tq, tk, tv, tdo, p2);
    // 5. back through rotation and norm; 6. gamma gradients
    mf::qk_prologue_bwd_kernel<D><<<pro_grid, mf::kPrologueThreads, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k),
        reinterpret_cast<const float4*>(dq_hat), reinterpret_cast<const float4*>(dk_hat), g_q_text,
        g_q_img, g_k_text, g_k_img, cu_seqlens_dev, segs_dev, n_samples, total_tokens, heads, eps,
        frame_dims, static_cast<uint4*>(dq), static_cast<uint4*>(dk), partial);
    const int n_out = 4 * D;
    mf::dgamma_reduce_kernel<<<(n_out + 31) / 32, 32 * mf::kReduceWarps, 0, s>>>(
        partial, bl.pro_blocks, n_out, dgamma);
    return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
  };
  if (head_dim == 128) return run(std::integral_constant<int, 128>{});
  return run(std::integral_constant<int, 64>{});
}

// --------------------------------------------------------- the sub-layer ---

namespace {

struct BlockLayout {
  WorkspaceLayout fwd;
  size_t x, v, o, rope, mods, total;
  int n_mtiles;
};

bool block_layout(int32_t total_tokens, int32_t heads, int32_t head_dim, BlockLayout* b) {
  if (!layout(total_tokens, heads, head_dim, &b->fwd)) return false;
  const size_t C = static_cast<size_t>(heads) * head_dim;
  const size_t mat = round_up(static_cast<size_t>(total_tokens) * C * 2, kAlign);
  b->n_mtiles = (total_tokens + mf::kGemmM - 1) / mf::kGemmM;
  b->x = round_up(b->fwd.total, kAlign);
  b->v = b->x + mat;
  b->o = b->v + mat;
  b->rope = b->o + mat;
  b->mods = b->rope + round_up(static_cast<size_t>(total_tokens) * (head_dim / 2) * 8, kAlign);
  b->total = b->mods + round_up(static_cast<size_t>(b->n_mtiles), kAlign);
  return true;
}

template <class Epi>
bool prepare_gemm_kernel() {
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(once[dev], [dev] {
    ok[dev] = cudaFuncSetAttribute(mf::gemm_kernel<Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mf::kGemmSmemBytes) == cudaSuccess;
  });
  return ok[dev];
}

}  // namespace

extern "C" size_t mf_block_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim) {
  BlockLayout b;
  return block_layout(total_tokens, heads, head_dim, &b) ? b.total : 0;
}

extern "C" mf_status mf_attn_block_fwd(
    const void* h, const float* shift, const float* scale, const float* gate, const void* w_qkv,
    const float* b_qkv, const void* w_o, const float* b_o, const float* g_q_text,
    const float* g_q_img, const float* g_k_text, const float* g_k_img,
    const int32_t* cu_seqlens_dev, const mf_segment* segs_dev, int32_t n_samples,
    const mf_work_item* work_dev, int32_t n_work, int32_t total_tokens, int32_t heads,
    int32_t head_dim, float eps_ln, float eps, int32_t frame_dims, float softmax_scale,
    void* h_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;
  const int64_t C = static_cast<int64_t>(heads) * head_dim;
  if (heads < 1 || C % 128 != 0 || C > mf::kAdalnMaxC) return MF_ERR_UNSUPPORTED;
  BlockLayout bl;
  if (!block_layout(total_tokens, heads, head_dim, &bl) || n_samples < 1 || n_work < 1)
    return MF_ERR_INVALID_ARG;
  if (!h || !shift || !scale || !gate || !w_qkv || !b_qkv || !w_o || !b_o || !g_q_text ||
      !g_q_img || !g_k_text || !g_k_img || !cu_seqlens_dev || !segs_dev || !work_dev || !h_out ||
      !workspace)
    return MF_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps) || !(eps_ln >= 0.0f) || !std::isfinite(eps_ln) ||
      !std::isfinite(softmax_scale))
    return MF_ERR_INVALID_ARG;
  if (frame_dims < 0 || frame_dims % 4 != 0 || frame_dims > head_dim - 4) return MF_ERR_INVALID_ARG;
  const void* al16[] = {h, shift, scale, gate, w_qkv, b_qkv, w_o, b_o, h_out};
  for (const void* ptr : al16)
    if (!aligned16(ptr)) return MF_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return MF_ERR_ALIGNMENT;
  if (workspace_bytes < bl.total) return MF_ERR_WORKSPACE;
  const size_t hb = static_cast<size_t>(total_tokens) * C * 2;
  if (overlaps(h_out, hb, h, hb) || overlaps(h_out, hb, workspace, bl.total))
    return MF_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* x = reinterpret_cast<__nv_bfloat16*>(ws + bl.x);
  auto* vb = reinterpret_cast<__nv_bfloat16*>(ws + bl.v);
  auto* ob = reinterpret_cast<__nv_bfloat16*>(ws + bl.o);
  auto* rope = reinterpret_cast<float2*>(ws + bl.rope);
  auto* mods = ws + bl.mods;
  const int sms = sm_count();
  if (sms <= 0) return MF_ERR_CUDA;

  CUtensorMap ta_x, tb_qkv, ta_o, tb_o;
  if (!encode_matrix(&ta_x, x, total_tokens, C, mf::kGemmM) ||
      !encode_matrix(&tb_qkv, w_qkv, 2 * 3 * C, C, mf::kGemmN) ||
      !encode_matrix(&ta_o, ob, total_tokens, C, mf::kGemmM) ||
      !encode_matrix(&tb_o, w_o, 2 * C, C, mf::kGemmN))
    return MF_ERR_CUDA;

  mf::GemmParams gp{};
  gp.rows = total_tokens;
  gp.k = static_cast<int>(C);
  gp.n_mtiles = bl.n_mtiles;
  gp.tile_mods = mods;
  gp.cu_seqlens = cu_seqlens_dev;
  gp.segs = segs_dev;
  gp.n_samples = n_samples;
  gp.heads = heads;
  gp.C = static_cast<int>(C);
  gp.eps = eps;
  gp.gammas[0] = g_q_text;
  gp.gammas[1] = g_q_img;
  gp.gammas[2] = g_k_text;
  gp.gammas[3] = g_k_img;
  gp.rope = rope;
  gp.q_hat = reinterpret_cast<__nv_bfloat16*>(ws + bl.fwd.q_hat);
  gp.k_hat = reinterpret_cast<__nv_bfloat16*>(ws + bl.fwd.k_hat);
  gp.v = vb;
  gp.h = static_cast<const __nv_bfloat16*>(h);
  gp.gate = gate;
  gp.h_out = static_cast<__nv_bfloat16*>(h_out);

  mf::tile_mods_kernel<<<bl.n_mtiles, mf::kGemmM, 0, s>>>(cu_seqlens_dev, segs_dev, n_samples,
                                                          total_tokens, mods);
  const int pairs = total_tokens * (head_dim / 2);
  if (head_dim == 128)
    mf::rope_table_kernel<128><<<(pairs + 255) / 256, 256, 0, s>>>(cu_seqlens_dev, segs_dev,
                                                                   n_samples, total_tokens,
                                                                   frame_dims, rope);
  else
    mf::rope_table_kernel<64><<<(pairs + 255) / 256, 256, 0, s>>>(cu_seqlens_dev, segs_dev,
                                                                  n_samples, total_tokens,
                                                                  frame_dims, rope);
  mf::adaln_kernel<<<(total_tokens + 7) / 8, 256, 0, s>>>(
      static_cast<const uint4*>(h), shift, scale, cu_seqlens_dev, segs_dev, n_samples,
      total_tokens, static_cast<int>(C), eps_ln, reinterpret_cast<uint4*>(x));

  // QKV projection with the QK-RMSNorm and rotation in its epilogue
  mf::GemmParams g1 = gp;
  g1.n_out = static_cast<int>(3 * C);
  g1.n_ntiles = static_cast<int>((3 * C + mf::kGemmN - 1) / mf::kGemmN);
  g1.bias = b_qkv;
  const int items1 = g1.n_mtiles * g1.n_ntiles;
  const unsigned grid1 = static_cast<unsigned>(items1 < sms ? items1 : sms);
  if (head_dim == 128) {
    if (!prepare_gemm_kernel<mf::EpiQkv<128>>()) return MF_ERR_CUDA;
    mf::gemm_kernel<mf::EpiQkv<128>><<<grid1, mf::kGemmThreads, mf::kGemmSmemBytes, s>>>(ta_x, tb_qkv, g1);
  } else {
    if (!prepare_gemm_kernel<mf::EpiQkv<64>>()) return MF_ERR_CUDA;
    mf::gemm_kernel<mf::EpiQkv<64>><<<grid1, mf::kGemmThreads, mf::kGemmSmemBytes, s>>>(ta_x, tb_qkv, g1);
  }
  if (cudaGetLastError() != cudaSuccess) return MF_ERR_CUDA;

  // the packed joint attention of q_hat, k_hat (already in the workspace) and v
  mf_status st = packed_attention_impl(vb, segs_dev, n_samples, work_dev, n_work, total_tokens,
                                       heads, head_dim, softmax_scale, ob, nullptr, workspace,
                                       bl.fwd.total, stream);
  if (st != MF_OK) return st;

  // output projection with bias, gate and residual in its epilogue
  mf::GemmParams g2 = gp;
  g2.n_out = static_cast<int>(C);
  g2.n_ntiles = static_cast<int>((C + mf::kGemmN - 1) / mf::kGemmN);
  g2.bias = b_o;
  const int items2 = g2.n_mtiles * g2.n_ntiles;
  const unsigned grid2 = static_cast<unsigned>(items2 < sms ? items2 : sms);
  if (!prepare_gemm_kernel<mf::EpiOut>()) return MF_ERR_CUDA;
  mf::gemm_kernel<mf::EpiOut><<<grid2, mf::kGemmThreads, mf::kGemmSmemBytes, s>>>(ta_o, tb_o, g2);
  return cudaGetLastError() == cudaSuccess ? MF_OK : MF_ERR_CUDA;
}
