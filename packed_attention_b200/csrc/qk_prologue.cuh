// Stage 1: modality-selected QK-RMSNorm + per-sample 2D RoPE.
//
// [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)":
//  modality-specific normalization before joint self-attention; video
//  overview, 00:03:16, and capabilities page, "Key Capabilities": per-sample
//  2D rotary embeddings on the latent grid.]
//
// For every token t and head h, and X in {q, k}:
//   x_hat = x * rsqrt(mean(x^2) + eps) * gamma_{X, modality(t)}
// then, for image tokens at grid (r, c), dims [0, d/2) rotate pairwise by
// r * theta_j and dims [d/2, d) by c * theta_j, theta_j = 10000^(-2j/(d/2)).
// Text tokens are not rotated. All arithmetic in fp32, one bf16 rounding.
//
// With frame_dims = F > 0 the rotation is 3D [same section, Conditioning:
// source and target latents told apart by a frame dimension of the RoPE]:
// dims [0, F) rotate by the token's frame index f (the sample's grids
// counted from 0), then two parts of S = (d - F) / 2 dims rotate by r and by
// c; each part uses theta_j = 10000^(-2j/width) with its own width (F or S).
// F = 0 is the 2D rotation above.
//
// HBM-bound: it reads q and k and writes q_hat and k_hat once (8 * T * H * d
// bytes). Layout of the work: one warp owns one token and walks its heads in
// groups of 32 / (d/8) (two heads at d = 128), each lane holding 8
// consecutive dims (one 16-byte vector) of q and of k, so every load and
// store instruction covers contiguous 512-byte spans. Each thread keeps the
// next kPrologueDepth groups of its q and k in flight with cp.async into its
// own shared-memory slots (no registers held, no barrier: a thread reads back
// only what it copied). The token's position, gammas and (cos, sin) pairs
// are computed once per token (theta of each pair once per block) and
// reused for all heads and for both q and k.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "bounds.cuh"
#include "packed_attention.cuh"
#include "sm100_ptx.cuh"

namespace mf {

// Threads per block of the per-token kernels (forward prologue, delta, norm
// backward).
constexpr int kPrologueThreads = 256;


__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
  uint4 v;
  v.x = pack_bf16x2(y[0], y[1]);
  v.y = pack_bf16x2(y[2], y[3]);
  v.z = pack_bf16x2(y[4], y[5]);
  v.w = pack_bf16x2(y[6], y[7]);
  return v;
}

// Where token t sits: text (no rotation) or its grid frame, row and column.
struct TokenPos {
  bool text;
  int frame, row, col;
};

__device__ __forceinline__ TokenPos token_position(const int32_t* __restrict__ cu_seqlens,
                                                   const mf_segment* __restrict__ segs,
                                                   int n_samples, int t) {
  // The sample that holds t: the last i with cu_seqlens[i] <= t.
  int lo = 0, hi = n_samples;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_seqlens + mid) <= t) lo = mid; else hi = mid;
  }
  const int j = t - __ldg(&segs[lo].start);
  const int n_text = __ldg(&segs[lo].n_text);
  TokenPos tp;
  tp.text = j < n_text;
  tp.frame = tp.row = tp.col = 0;
  if (!tp.text) {
    const int gw = __ldg(&segs[lo].grid_w);
    const int hw = __ldg(&segs[lo].grid_h) * gw;
    const int p = (j - n_text) % hw;  // every frame of a sample shares the grid positions
    tp.frame = (j - n_text) / hw;
    tp.row = p / gw;
    tp.col = p % gw;
  }
  return tp;
}

// theta_j = 10000^(-2j/width) = 2^(-(2j/width) * log2(10000)) for the pair
// whose first dim is `e` dims into a part of `width` dims.
__device__ __forceinline__ double pair_theta(int e, int width) {
  constexpr double kLog2Base = 13.287712379549449;
  return exp2(-(2.0 * (e / 2) / width) * kLog2Base);
}

// (cos, sin) of pos * theta: the angle is formed and reduced to [-pi, pi] in
// fp64, so the fp32 sine and cosine see an argument accurate to ~1e-7 rad
// however large the grid position is.
__device__ __forceinline__ float2 rotation_cos_sin(int pos, double theta) {
  constexpr double kTwoPi = 6.283185307179586;
  constexpr double kInvTwoPi = 0.15915494309189535;
  double ang = static_cast<double>(pos) * theta;
  ang -= kTwoPi * rint(ang * kInvTwoPi);
  float sn, cs;
  sincosf(static_cast<float>(ang), &sn, &cs);
  return make_float2(cs, sn);
}

// Which grid coordinate turns pair `pair` (0 frame, 1 row, 2 column), and
// the pair's first dim within its part and the part's width.
__device__ __forceinline__ int pair_axis(int pair, int d, int frame_dims, int& e_in, int& width) {
  const int spatial = (d - frame_dims) / 2;
  const int e = 2 * pair;
  if (e < frame_dims) { e_in = e; width = frame_dims; return 0; }
  if (e < frame_dims + spatial) { e_in = e - frame_dims; width = spatial; return 1; }
  e_in = e - frame_dims - spatial;
  width = spatial;
  return 2;
}

// (cos, sin) of rotation pair `pair` (dims 2*pair, 2*pair + 1) of a token at
// `tp`. Every kernel that rotates (forward, backward, sub-layer) takes its
// angles from these helpers.
template <int D>
__device__ __forceinline__ float2 pair_cos_sin(const TokenPos& tp, int pair, int frame_dims) {
  if (tp.text) return make_float2(1.0f, 0.0f);
  int e_in, width;
  const int axis = pair_axis(pair, D, frame_dims, e_in, width);
  const int pos = axis == 0 ? tp.frame : (axis == 1 ? tp.row : tp.col);
  return rotation_cos_sin(pos, pair_theta(e_in, width));
}

// Tokens of a forward prologue block: one per warp.
constexpr int kPrologueTokPerBlock = kPrologueThreads / 32;
// Head groups of q and k in flight per thread.
constexpr int kPrologueDepth = 5;

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4) qk_prologue_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const float* __restrict__ gq_text,
    const float* __restrict__ gq_img, const float* __restrict__ gk_text,
    const float* __restrict__ gk_img, const int32_t* __restrict__ cu_seqlens,
    const mf_segment* __restrict__ segs, int n_samples, int total_tokens, int heads, float eps,
    int frame_dims, uint4* __restrict__ q_hat, uint4* __restrict__ k_hat) {
  constexpr int kVecPerRow = D / 8;       // 16-byte vectors per row
  constexpr int kRows = 32 / kVecPerRow;  // heads one warp instruction covers
  constexpr int kP = kPrologueDepth;
  __shared__ double s_theta[D / 2];
  __shared__ int32_t s_axis[D / 2];
  // Per thread: its 16 bytes of q and of k for kP head groups ahead.
  __shared__ uint4 ring[kP][2][kPrologueThreads];

  const int lane = threadIdx.x % 32;
  const int vec = lane % kVecPerRow;
  const int hsub = lane / kVecPerRow;  // head within each group of kRows
  const int t_raw = blockIdx.x * kPrologueTokPerBlock + threadIdx.x / 32;
  // A warp past the last token computes on a valid token and stores nothing.
  const bool active = t_raw < total_tokens;
  const int t = active ? t_raw : total_tokens - 1;
  // Lane l holds vector l of the token's rows g*kRows .. g*kRows + kRows - 1:
  // each instruction moves kRows * 2 * D contiguous bytes.
  const size_t base = static_cast<size_t>(t) * heads * kVecPerRow + lane;
  const long long n_vec = static_cast<long long>(total_tokens) * heads * kVecPerRow;
  const int n_groups = (heads + kRows - 1) / kRows;

  // The first kP groups are requested before any setup; every iteration
  // commits one group of copies (empty past the end), so group g is always
  // the (g+1)-th commit.
#pragma unroll
  for (int i = 0; i < kP; ++i) {
    const size_t gi = base + static_cast<size_t>(i) * kRows * kVecPerRow;
    if (i * kRows + hsub < heads && in_bounds(gi, n_vec)) {
      cp_async16(&ring[i][0][threadIdx.x], q + gi);
      cp_async16(&ring[i][1][threadIdx.x], k + gi);
    }
    cp_async_commit();
  }
  // theta and axis of every pair, once per block
  for (int pr = threadIdx.x; pr < D / 2; pr += kPrologueThreads) {
    int e_in, width;
    s_axis[pr] = pair_axis(pr, D, frame_dims, e_in, width);
    s_theta[pr] = pair_theta(e_in, width);
  }
  __syncthreads();

  // The token's position, gammas and the (cos, sin) of the 4 pairs of a
  // lane's 8 dims: once per token, for all heads and for both q and k. The
  // kRows lanes that own the same dims compute 4 / kRows pairs each and swap.
  const TokenPos tp = token_position(cu_seqlens, segs, n_samples, t);
  const int e0 = vec * 8;  // first dim this lane owns
  float cs[4], sn[4];
  {
    float rc[4 / kRows], rs[4 / kRows];
#pragma unroll
    for (int ii = 0; ii < 4 / kRows; ++ii) {
      const int pair = e0 / 2 + ii * kRows + hsub;
      float2 r = make_float2(1.0f, 0.0f);
      if (!tp.text) {
        const int axis = s_axis[pair];
        r = rotation_cos_sin(axis == 0 ? tp.frame : (axis == 1 ? tp.row : tp.col), s_theta[pair]);
      }
      rc[ii] = r.x;
      rs[ii] = r.y;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int src = (i % kRows) * kVecPerRow + vec;
      cs[i] = __shfl_sync(0xffffffffu, rc[i / kRows], src);
      sn[i] = __shfl_sync(0xffffffffu, rs[i / kRows], src);
    }
  }
  float gq[8], gk[8];
  {
    const float* gqs = tp.text ? gq_text : gq_img;
    const float* gks = tp.text ? gk_text : gk_img;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      gq[i] = __ldg(gqs + e0 + i);
      gk[i] = __ldg(gks + e0 + i);
    }
  }

  const float inv_d = 1.0f / D;
  for (int g = 0; g < n_groups; ++g) {
    const int h = g * kRows + hsub;
    const bool head_in = h < heads;  // the last group may be partial
    const size_t idx = base + static_cast<size_t>(g) * kRows * kVecPerRow;
    const int slot = g % kP;
    cp_async_wait<kP - 1>();  // group g has landed
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4 qv = head_in ? ring[slot][0][threadIdx.x] : zero;
    const uint4 kv = head_in ? ring[slot][1][threadIdx.x] : zero;
    float xq[8], xk[8];
    unpack8(qv, xq);
    unpack8(kv, xk);
    float ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ssq = fmaf(xq[i], xq[i], ssq);
      ssk = fmaf(xk[i], xk[i], ssk);
    }
#pragma unroll
    for (int o = kVecPerRow / 2; o > 0; o >>= 1) {
      ssq += __shfl_xor_sync(0xffffffffu, ssq, o, kVecPerRow);
      ssk += __shfl_xor_sync(0xffffffffu, ssk, o, kVecPerRow);
    }
    const float rq = rsqrtf(fmaf(ssq, inv_d, eps));
    const float rk = rsqrtf(fmaf(ssk, inv_d, eps));
    float yq[8], yk[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float qa = xq[2 * i] * rq * gq[2 * i], qb = xq[2 * i + 1] * rq * gq[2 * i + 1];
      const float ka = xk[2 * i] * rk * gk[2 * i], kb = xk[2 * i + 1] * rk * gk[2 * i + 1];
      yq[2 * i] = qa * cs[i] - qb * sn[i];
      yq[2 * i + 1] = qa * sn[i] + qb * cs[i];
      yk[2 * i] = ka * cs[i] - kb * sn[i];
      yk[2 * i + 1] = ka * sn[i] + kb * cs[i];
    }
    if (active && head_in && in_bounds(idx, n_vec)) {
      q_hat[idx] = pack8(yq);
      k_hat[idx] = pack8(yk);
    }
    // The slot's values are in registers and used above: refill it with
    // group g + kP.
    const size_t gi = idx + static_cast<size_t>(kP) * kRows * kVecPerRow;
    if (h + kP * kRows < heads && in_bounds(gi, n_vec)) {
      cp_async16(&ring[slot][0][threadIdx.x], q + gi);
      cp_async16(&ring[slot][1][threadIdx.x], k + gi);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
}

}  // namespace mf
