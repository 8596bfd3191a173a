// The HBM-bound passes of the backward: D = rowsum(dO * out), and the
// gradients through the RMSNorm and the rotation with the gamma gradients.
//
// [Chain rule through the forward prologue (Mage-Flow paper summary,
//  "Native-Resolution MMDiT (NR-MMDiT)": modality-specific normalization,
//  2D/3D rotary embeddings).] For one (token, head) row x of q or k, with
// r = rsqrt(mean(x^2) + eps), x_n = x * r, the forward gave
// x_hat = R(pos) (x_n * gamma). Given dx_hat:
//   dy      = R(pos)^T dx_hat             (text tokens: dy = dx_hat)
//   dgamma += dy * x_n                    (per role q/k and modality)
//   dx      = r * (dy * gamma - x_n * (x_n . (dy * gamma)) / d)
//
// Layout of work: d/8 threads own one token and loop over its heads, 16-byte
// vectors; the token's rotation is set up once.
// The gamma gradients are reduced without atomics: per block in a fixed
// order into a partial row, then over blocks in a fixed order, so that the
// result is the same on every run.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "qk_prologue.cuh"

namespace mf {

// D[h, t] = sum_m dO[t, h, m] * out[t, h, m] in fp32.
template <int D>
__global__ void __launch_bounds__(kPrologueThreads) bwd_delta_kernel(
    const uint4* __restrict__ out, const uint4* __restrict__ dout, int total_tokens, int heads,
    float* __restrict__ delta) {
  constexpr int kVecPerRow = D / 8;
  constexpr int kTokPerBlock = kPrologueThreads / kVecPerRow;
  const int vec = threadIdx.x % kVecPerRow;
  const int t_raw = blockIdx.x * kTokPerBlock + threadIdx.x / kVecPerRow;
  const bool active = t_raw < total_tokens;
  const int t = active ? t_raw : total_tokens - 1;
  const size_t row0 = static_cast<size_t>(t) * heads * kVecPerRow + vec;
  const long long n_vec = static_cast<long long>(total_tokens) * heads * kVecPerRow;
  for (int h = 0; h < heads; ++h) {
    const size_t idx = row0 + static_cast<size_t>(h) * kVecPerRow;
    const bool in = in_bounds(idx, n_vec);
    float a[8], b[8];
    unpack8(in ? __ldg(out + idx) : make_uint4(0, 0, 0, 0), a);
    unpack8(in ? __ldg(dout + idx) : make_uint4(0, 0, 0, 0), b);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(a[i], b[i], s);
#pragma unroll
    for (int o = kVecPerRow / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o, kVecPerRow);
    const size_t di = static_cast<size_t>(h) * total_tokens + t;
    if (active && vec == 0 && in_bounds(di, static_cast<long long>(heads) * total_tokens))
      delta[di] = s;
  }
}

// The (cos, sin) of the 4 pairs a thread owns, for token t (text: identity),
// from the forward prologue's positions and angles; returns whether t is text.
template <int D>
__device__ __forceinline__ bool token_rotation(const int32_t* __restrict__ cu_seqlens,
                                               const mf_segment* __restrict__ segs, int n_samples,
                                               int t, int e0, int frame_dims, float (&cs)[4],
                                               float (&sn)[4]) {
  const TokenPos tp = token_position(cu_seqlens, segs, n_samples, t);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 r = pair_cos_sin<D>(tp, e0 / 2 + i, frame_dims);
    cs[i] = r.x;
    sn[i] = r.y;
  }
  return tp.text;
}

// dq, dk (bf16) from dq_hat, dk_hat (fp32) and the raw q, k; partial gamma
// gradients per block: partial[block][4][D] in the order q_text, q_img,
// k_text, k_img.
template <int D>
__global__ void __launch_bounds__(kPrologueThreads) qk_prologue_bwd_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const float4* __restrict__ dq_hat,
    const float4* __restrict__ dk_hat, const float* __restrict__ gq_text,
    const float* __restrict__ gq_img, const float* __restrict__ gk_text,
    const float* __restrict__ gk_img, const int32_t* __restrict__ cu_seqlens,
    const mf_segment* __restrict__ segs, int n_samples, int total_tokens, int heads, float eps,
    int frame_dims, uint4* __restrict__ dq, uint4* __restrict__ dk, float* __restrict__ partial) {
  constexpr int kVecPerRow = D / 8;
  constexpr int kTokPerBlock = kPrologueThreads / kVecPerRow;
  __shared__ float s_red[kTokPerBlock][2][D];
  __shared__ int s_text[kTokPerBlock];

  const int vec = threadIdx.x % kVecPerRow;
  const int tok = threadIdx.x / kVecPerRow;
  const int t_raw = blockIdx.x * kTokPerBlock + tok;
  const bool active = t_raw < total_tokens;
  const int t = active ? t_raw : total_tokens - 1;
  const int e0 = vec * 8;
  float cs[4], sn[4];
  const bool is_text = token_rotation<D>(cu_seqlens, segs, n_samples, t, e0, frame_dims, cs, sn);

  float gq[8], gk[8];
  {
    const float* gqs = is_text ? gq_text : gq_img;
    const float* gks = is_text ? gk_text : gk_img;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      gq[i] = __ldg(gqs + e0 + i);
      gk[i] = __ldg(gks + e0 + i);
    }
  }
  float accq[8], acck[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) accq[i] = acck[i] = 0.f;

  const float inv_d = 1.0f / D;
  const size_t row0 = static_cast<size_t>(t) * heads * kVecPerRow + vec;
  const long long n_vec = static_cast<long long>(total_tokens) * heads * kVecPerRow;
#pragma unroll 1
  for (int h = 0; h < heads; ++h) {
    const size_t idx = row0 + static_cast<size_t>(h) * kVecPerRow;
    const bool in = in_bounds(idx, n_vec);  // covers dq_hat / dk_hat's 2 * idx + 1 too
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      float x[8], dy[8];
      unpack8(in ? __ldg((which ? k : q) + idx) : make_uint4(0, 0, 0, 0), x);
      const float4* dh = which ? dk_hat : dq_hat;
      const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 d0 = in ? __ldg(dh + 2 * idx) : z4, d1 = in ? __ldg(dh + 2 * idx + 1) : z4;
      const float dx_hat[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      // transposed rotation: (a, b) -> (a cos + b sin, -a sin + b cos)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = dx_hat[2 * i], b = dx_hat[2 * i + 1];
        dy[2 * i] = a * cs[i] + b * sn[i];
        dy[2 * i + 1] = b * cs[i] - a * sn[i];
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
      for (int o = kVecPerRow / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, kVecPerRow);
      const float r = rsqrtf(fmaf(ss, inv_d, eps));
      const float* g = which ? gk : gq;
      float* acc = which ? acck : accq;
      float xn[8], dxn[8], dot = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        xn[i] = x[i] * r;
        acc[i] = fmaf(dy[i], xn[i], acc[i]);
        dxn[i] = dy[i] * g[i];
        dot = fmaf(xn[i], dxn[i], dot);
      }
#pragma unroll
      for (int o = kVecPerRow / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o, kVecPerRow);
      const float c = dot * inv_d;
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = r * fmaf(-xn[i], c, dxn[i]);
      if (active && in) (which ? dk : dq)[idx] = pack8(y);
    }
  }

  // ---- gamma gradients: this block's partial row, in a fixed order ----
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_red[tok][0][e0 + i] = active ? accq[i] : 0.f;
    s_red[tok][1][e0 + i] = active ? acck[i] : 0.f;
  }
  if (vec == 0) s_text[tok] = is_text ? 1 : 0;
  __syncthreads();
  for (int o = threadIdx.x; o < 4 * D; o += kPrologueThreads) {
    const int which = o / (2 * D);           // 0: q, 1: k
    const int want_text = (o / D) % 2 == 0;  // order q_text, q_img, k_text, k_img
    const int m = o % D;
    float s = 0.f;
    for (int tk = 0; tk < kTokPerBlock; ++tk)
      if (s_text[tk] == want_text) s += s_red[tk][which][m];
    const size_t pi = static_cast<size_t>(blockIdx.x) * 4 * D + o;
    if (in_bounds(pi, static_cast<long long>(gridDim.x) * 4 * D)) partial[pi] = s;
  }
}

// dgamma[o] = sum over blocks of partial[b][o]. A CTA of 8 warps owns 32
// outputs (one per lane); warp w sums the w-th contiguous eighth of the
// blocks, then the eight partial sums are added in warp order: a fixed
// order, so the result is the same on every run.
constexpr int kReduceWarps = 8;

__global__ void __launch_bounds__(32 * kReduceWarps) dgamma_reduce_kernel(
    const float* __restrict__ partial, int n_blocks, int n_out, float* __restrict__ dgamma) {
  __shared__ float s_part[kReduceWarps][32];
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  const int o = blockIdx.x * 32 + lane;
  const int per = (n_blocks + kReduceWarps - 1) / kReduceWarps;
  const int b0 = w * per, b1 = min(n_blocks, b0 + per);
  float s = 0.f;
  if (o < n_out)
    for (int b = b0; b < b1; ++b) {
      const size_t pi = static_cast<size_t>(b) * n_out + o;
      if (in_bounds(pi, static_cast<long long>(n_blocks) * n_out)) s += __ldg(partial + pi);
    }
  s_part[w][lane] = s;
  __syncthreads();
  if (w == 0 && o < n_out) {
    float t = 0.f;
    for (int i = 0; i < kReduceWarps; ++i) t += s_part[i][lane];
    dgamma[o] = t;
  }
}

}  // namespace mf
