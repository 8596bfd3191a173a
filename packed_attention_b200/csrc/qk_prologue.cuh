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
// bytes), a copy-shaped stream. Persistent: one CTA per SM takes a
// contiguous range of chunks of `tps` tokens (every head of a token is one
// contiguous H*d*2-byte row of q and of k).
//   warp 8 (1 lane)  producer: bulk-copies each chunk's q and k rows into a
//                    ring of shared-memory stages (one mbarrier per stage,
//                    completion counted in bytes), so that many chunks are
//                    in flight however long the math takes.
//   warps 0-7        each on its own chunks (warp w of W: the CTA's chunks
//                    w, w + W, ..., in stages of its own): first the (cos, sin) of every rotation
//                    pair of the chunk's tokens into the warp's small shared
//                    table (one sincos per pair and token, not per head),
//                    then each (token, head) row of q and k: d/8 lanes per
//                    row, 8 consecutive dims (one 16-byte vector) each, the
//                    mean square by shuffles within the row's lanes; 16-byte
//                    stores of q_hat, k_hat that cover whole 512-byte row
//                    pairs per warp.
// Every wait is bounded; a wait that runs out records MF_ERR_TIMEOUT, every
// warp leaves its loop, and the producer waits (bounded) for its copies in
// flight.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "bounds.cuh"
#include "packed_attention.cuh"
#include "sm100_ptx.cuh"

namespace mf {

// Threads per block of the backward's per-token kernels (delta, norm backward).
constexpr int kPrologueThreads = 256;

constexpr int kProComputeThreads = 256;  // warps 0-7
constexpr int kProThreads = kProComputeThreads + 32;
constexpr int kProMaxStages = 16;
constexpr int kProMaxTps = 16;
constexpr int kProSmemBudget = 200 * 1024;  // stages + tables, below the 227 KB per CTA

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

// Chunking and staging of one launch, chosen on the host.
struct ProloguePlan {
  int tps;     // tokens per chunk
  int stages;  // ring depth, a multiple of warps
  int warps;   // compute warps in use (<= 8); warp w owns stages w, w + warps, ...
};

__host__ __device__ constexpr size_t prologue_stage_bytes(int tps, int heads, int d) {
  return 2 * static_cast<size_t>(tps) * heads * d * 2;  // q rows, then k rows
}

// Per compute warp: the (cos, sin) of every pair of its chunk's tokens, then
// their text flags.
__host__ __device__ constexpr size_t prologue_table_bytes(int tps, int d) {
  return static_cast<size_t>(tps) * (d / 2) * 8 + kProMaxTps * 4;
}

__host__ __device__ constexpr size_t prologue_smem_bytes(ProloguePlan pp, int heads, int d) {
  return pp.stages * prologue_stage_bytes(pp.tps, heads, d) +
         (kProComputeThreads / 32) * prologue_table_bytes(pp.tps, d);
}

template <int D>
__global__ void __launch_bounds__(kProThreads, 1) qk_prologue_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const float* __restrict__ gq_text,
    const float* __restrict__ gq_img, const float* __restrict__ gk_text,
    const float* __restrict__ gk_img, const int32_t* __restrict__ cu_seqlens,
    const mf_segment* __restrict__ segs, int n_samples, int total_tokens, int heads, float eps,
    int frame_dims, ProloguePlan plan, uint4* __restrict__ q_hat, uint4* __restrict__ k_hat) {
  constexpr int kTpr = D / 8;              // threads (16-byte vectors) per row
  constexpr int kRowsPerPass = 32 / kTpr;  // rows a warp handles at once
  constexpr int kWarps = kProComputeThreads / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kProMaxStages], empty[kProMaxStages];
  __shared__ double s_theta[D / 2];
  __shared__ int32_t s_axis[D / 2];
  __shared__ int32_t abort_word;
  volatile int32_t* abort_flag = &abort_word;

  const int tps = plan.tps, S = plan.stages, W = plan.warps;
  const size_t tok_bytes = static_cast<size_t>(heads) * D * 2;
  const size_t stage_bytes = prologue_stage_bytes(tps, heads, D);

  const int n_chunks = (total_tokens + tps - 1) / tps;
  const int c0 = static_cast<int>(static_cast<long long>(blockIdx.x) * n_chunks / gridDim.x);
  const int c1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * n_chunks / gridDim.x);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    abort_word = 0;
    fence_mbarrier_init();
  }
  // theta and axis of every pair, once per CTA
  for (int pr = threadIdx.x; pr < D / 2; pr += blockDim.x) {
    int e_in, width;
    s_axis[pr] = pair_axis(pr, D, frame_dims, e_in, width);
    s_theta[pr] = pair_theta(e_in, width);
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------------------------------------------------- producer ---
    if (lane == 0) {
      const size_t tensor_bytes = static_cast<size_t>(total_tokens) * tok_bytes;
      int i = 0;
      bool ok = true;
      for (int c = c0; c < c1; ++c, ++i) {
        const int s = i % S;
        if (i >= S && !wait_bar(&empty[s], ((i / S) - 1) & 1, abort_flag)) { ok = false; break; }
        const int t0 = c * tps;
        const int ntok = min(tps, total_tokens - t0);
        const uint32_t bytes = static_cast<uint32_t>(ntok * tok_bytes);
        const uint8_t* src_q = reinterpret_cast<const uint8_t*>(q) + t0 * tok_bytes;
        const uint8_t* src_k = reinterpret_cast<const uint8_t*>(k) + t0 * tok_bytes;
        if (!in_span(src_q, bytes, q, tensor_bytes) || !in_span(src_k, bytes, k, tensor_bytes)) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_load(smem + s * stage_bytes, src_q, bytes, &full[s]);
        bulk_load(smem + s * stage_bytes + tps * tok_bytes, src_k, bytes, &full[s]);
      }
      if (!ok) {
        // Every copy already issued must land before the CTA exits: wait for
        // the stages of the last min(i, S) chunks (earlier ones were consumed).
        for (int j = i - S > 0 ? i - S : 0; j < i; ++j)
          wait_slow(&full[j % S], (j / S) & 1, nullptr, kDrainLimitNs);
      }
    }
    return;
  }

  // ------------------------------------------------------------- compute ---
  // Warp w takes this CTA's chunks w, w + W, w + 2W, ... on its own: the
  // rotation table of its chunk, then the chunk's 2 * tokens * heads rows.
  // Chunk i sits in stage i % S and S is a multiple of W, so a stage only
  // ever holds one warp's chunks, in that warp's order: each parity wait is
  // on the phase right after the one the warp consumed last.
  if (warp >= W) return;
  const int vec = lane % kTpr;
  const int e0 = vec * 8;  // first dim this thread owns
  float g[4][8];           // q_text, q_img, k_text, k_img: this thread's 8 dims
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    g[0][m] = __ldg(gq_text + e0 + m);
    g[1][m] = __ldg(gq_img + e0 + m);
    g[2][m] = __ldg(gk_text + e0 + m);
    g[3][m] = __ldg(gk_img + e0 + m);
  }
  float2* table = reinterpret_cast<float2*>(smem + S * stage_bytes +
                                            warp * prologue_table_bytes(tps, D));
  int32_t* text = reinterpret_cast<int32_t*>(table + tps * (D / 2));
  const float inv_d = 1.0f / D;
  const long long n_vec = static_cast<long long>(total_tokens) * heads * kTpr;
  for (int i = warp; c0 + i < c1; i += W) {
    const int s = i % S;
    if (!warp_wait_bar(&full[s], (i / S) & 1, abort_flag)) break;
    const int t0 = (c0 + i) * tps;
    const int ntok = min(tps, total_tokens - t0);
    // (cos, sin) of every pair of every token of the chunk, and its modality.
    for (int pr = lane; pr < ntok * (D / 2); pr += 32) {
      const int tl = pr / (D / 2), pair = pr % (D / 2);
      const TokenPos tp = token_position(cu_seqlens, segs, n_samples, t0 + tl);
      if (tp.text) {
        table[pr] = make_float2(1.0f, 0.0f);
      } else {
        const int axis = s_axis[pair];
        table[pr] = rotation_cos_sin(axis == 0 ? tp.frame : (axis == 1 ? tp.row : tp.col),
                                     s_theta[pair]);
      }
      if (pair == 0) text[tl] = tp.text ? 1 : 0;
    }
    __syncwarp();
    const uint8_t* stage = smem + s * stage_bytes;
    const int rows = 2 * ntok * heads;  // q rows of the chunk, then its k rows
    const int rows_q = ntok * heads;
#pragma unroll 4
    for (int r0 = 0; r0 < rows; r0 += kRowsPerPass) {
      const int r = r0 + lane / kTpr;
      const bool valid = r < rows;
      // A row past the chunk's end computes on its last row (so that every
      // thread of the row group takes part in the shuffles) and stores nothing.
      const int re = valid ? r : rows - 1;
      const int kk = re >= rows_q;      // 0: q, 1: k
      const int rr = re - kk * rows_q;  // (token, head) row within the chunk
      const int tl = rr / heads;
      float x[8];
      unpack8(*reinterpret_cast<const uint4*>(stage + kk * tps * tok_bytes +
                                              static_cast<size_t>(rr) * D * 2 + vec * 16),
              x);
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) ss = fmaf(x[m], x[m], ss);
#pragma unroll
      for (int o = kTpr / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, kTpr);
      const float rn = rsqrtf(fmaf(ss, inv_d, eps));
      const bool tx = text[tl] != 0;
      float gm[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) gm[m] = kk ? (tx ? g[2][m] : g[3][m]) : (tx ? g[0][m] : g[1][m]);
      const float4 cs01 = *reinterpret_cast<const float4*>(table + tl * (D / 2) + 4 * vec);
      const float4 cs23 = *reinterpret_cast<const float4*>(table + tl * (D / 2) + 4 * vec + 2);
      const float cs[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
      const float sn[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
      float y[8];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float a = x[2 * m] * rn * gm[2 * m], b = x[2 * m + 1] * rn * gm[2 * m + 1];
        y[2 * m] = a * cs[m] - b * sn[m];
        y[2 * m + 1] = a * sn[m] + b * cs[m];
      }
      const size_t idx = (static_cast<size_t>(t0) * heads + rr) * kTpr + vec;
      if (valid && in_bounds(idx, n_vec)) (kk ? k_hat : q_hat)[idx] = pack8(y);
    }
    // This warp is done with the stage and its table.
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace mf
