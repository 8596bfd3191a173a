// The joint-attention sub-layer around the packed path: adaLN modulation,
// per-modality QKV projection with the QK-RMSNorm and RoPE fused into its
// epilogue, and per-modality output projection with bias, gate and residual
// fused into its epilogue.
//
// [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": an MMDiT
//  (text and image streams with their own parameters) with modality-specific
//  normalization and joint self-attention; "Training Infrastructure": the
//  adaptive normalization / RoPE / gating chains fused into CUDA kernels.]
// For token t of sample s and modality m (0 text, 1 image):
//   x_t  = LN(h_t) * (1 + scale[s, m]) + shift[s, m]     adaln_kernel
//   qkv  = W_qkv[m] x_t + b_qkv[m]                       gemm_kernel<EpiQkv>: q, k
//          go straight through RMSNorm (per head) and the rotation to q_hat,
//          k_hat; v is stored as is
//   o    = packed joint attention                        packed_attention_kernel
//   h'_t = h_t + gate[s, m] * (W_o[m] o_t + b_o[m])      gemm_kernel<EpiOut>
//
// The GEMM: persistent, one CTA per SM, tiles of 128 rows x 256 columns,
// K in steps of 64 through a 4-stage TMA ring (A: 128 x 64, B: 256 x 64,
// 128-byte swizzle), tcgen05 MMAs (M = 128, N = 256, K = 16) into one of two
// TMEM accumulators (256 columns each), so that the epilogue of one tile
// overlaps the MMAs of the next. A 128-row tile holding tokens of both
// modalities is computed twice, once per weight matrix, and each pass stores
// only its modality's rows. Tiles are taken row-major (all column tiles of a
// row tile, then the next) so that an A tile is read from HBM once and the
// weights stay in L2.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "packed_attention.cuh"
#include "qk_prologue.cuh"

namespace mf {

constexpr int kGemmThreads = 320;       // 8 epilogue warps, producer, MMA issuer
constexpr int kGemmProducerWarp = 8;
constexpr int kGemmMmaWarp = 9;
constexpr int kGemmM = 128, kGemmN = 256, kGemmK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = kGemmM * kGemmK * 2;  // 16 KB
constexpr int kGemmBBytes = kGemmN * kGemmK * 2;  // 32 KB
constexpr int kGemmSmemBytes = kGemmStages * (kGemmABytes + kGemmBBytes) + 1024;

// Sample and modality of token t (0 text, 1 image); cu_seqlens as planned.
__device__ __forceinline__ void token_sample_mod(const int32_t* __restrict__ cu_seqlens,
                                                 const mf_segment* __restrict__ segs,
                                                 int n_samples, int t, int& s, int& m) {
  int lo = 0, hi = n_samples;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_seqlens + mid) <= t) lo = mid; else hi = mid;
  }
  s = lo;
  m = (t - __ldg(&segs[lo].start)) < __ldg(&segs[lo].n_text) ? 0 : 1;
}

// ------------------------------------------------------------- adaLN ---

// One warp per token: two-pass mean and variance over the C channels in
// registers (C <= kAdalnMaxC, a multiple of 8), then the modulation.
constexpr int kAdalnMaxC = 4096;

__global__ void __launch_bounds__(256) adaln_kernel(
    const uint4* __restrict__ h, const float* __restrict__ shift, const float* __restrict__ scale,
    const int32_t* __restrict__ cu_seqlens, const mf_segment* __restrict__ segs, int n_samples,
    int total_tokens, int C, float eps, uint4* __restrict__ x) {
  constexpr int kMaxV = kAdalnMaxC / 8 / 32;  // 16-byte vectors per lane
  const int lane = threadIdx.x % 32;
  const int t = blockIdx.x * 8 + threadIdx.x / 32;
  if (t >= total_tokens) return;
  int s, m;
  token_sample_mod(cu_seqlens, segs, n_samples, t, s, m);
  const int nv = C / 8;
  const uint4* row = h + static_cast<size_t>(t) * nv;
  float v[kMaxV][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxV; ++i) {
    const int vi = lane + 32 * i;
    if (vi < nv) {
      unpack8(__ldg(row + vi), v[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += v[i][e];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / C;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxV; ++i)
    if (lane + 32 * i < nv) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dlt = v[i][e] - mean;
        sq = fmaf(dlt, dlt, sq);
      }
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / C + eps);
  const size_t mod_row = (static_cast<size_t>(s) * 2 + m) * C;
  uint4* out = x + static_cast<size_t>(t) * nv;
#pragma unroll
  for (int i = 0; i < kMaxV; ++i) {
    const int vi = lane + 32 * i;
    if (vi < nv) {
      const float4* sh = reinterpret_cast<const float4*>(shift + mod_row) + 2 * vi;
      const float4* sc = reinterpret_cast<const float4*>(scale + mod_row) + 2 * vi;
      const float4 a0 = __ldg(sh), a1 = __ldg(sh + 1), b0 = __ldg(sc), b1 = __ldg(sc + 1);
      const float shv[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float scv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = fmaf((v[i][e] - mean) * rstd, 1.0f + scv[e], shv[e]);
      out[vi] = pack8(y);
    }
  }
}

// ------------------------------------------- rotation table, tile masks ---

// (cos, sin) of every rotation pair of every token, [T, D/2]: the forward
// prologue's positions and angle formation; text tokens get (1, 0).
template <int D>
__global__ void rope_table_kernel(const int32_t* __restrict__ cu_seqlens,
                                  const mf_segment* __restrict__ segs, int n_samples,
                                  int total_tokens, int frame_dims, float2* __restrict__ table) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_tokens * (D / 2)) return;
  const int t = idx / (D / 2), pair = idx % (D / 2);
  table[idx] = pair_cos_sin<D>(token_position(cu_seqlens, segs, n_samples, t), pair, frame_dims);
}

// Per 128-row tile: bit 0 if it holds text tokens, bit 1 if image tokens.
__global__ void __launch_bounds__(kGemmM) tile_mods_kernel(
    const int32_t* __restrict__ cu_seqlens, const mf_segment* __restrict__ segs, int n_samples,
    int total_tokens, uint8_t* __restrict__ mods) {
  __shared__ int mask;
  if (threadIdx.x == 0) mask = 0;
  __syncthreads();
  const int t = blockIdx.x * kGemmM + threadIdx.x;
  if (t < total_tokens) {
    int s, m;
    token_sample_mod(cu_seqlens, segs, n_samples, t, s, m);
    atomicOr(&mask, 1 << m);
  }
  __syncthreads();
  if (threadIdx.x == 0) mods[blockIdx.x] = static_cast<uint8_t>(mask);
}

// ------------------------------------------------------------- GEMM ---

struct GemmParams {
  int rows;         // T
  int n_out;        // output columns per modality (3C or C)
  int k;            // reduction length (C)
  int n_mtiles, n_ntiles;
  const uint8_t* tile_mods;
  const int32_t* cu_seqlens;
  const mf_segment* segs;
  int n_samples;
  const float* bias;      // [2, n_out]
  // EpiQkv
  int heads, C;
  float eps;
  const float* gammas[4];  // q_text, q_img, k_text, k_img
  const float2* rope;      // [T, D/2]
  __nv_bfloat16* q_hat;    // [T, H, D]
  __nv_bfloat16* k_hat;
  __nv_bfloat16* v;
  // EpiOut
  const __nv_bfloat16* h;  // [T, C] residual
  const float* gate;       // [n, 2, C]
  __nv_bfloat16* h_out;
};

struct GemmCtl {
  uint64_t full[kGemmStages], empty[kGemmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
};

// Passes of a work item: one per modality present in its row tile.
__device__ __forceinline__ int gemm_passes(const GemmParams& p, int item, int* mods) {
  const int mt = item / p.n_ntiles;
  const int mask = p.tile_mods[mt];
  int n = 0;
  if (mask & 1) mods[n++] = 0;
  if (mask & 2) mods[n++] = 1;
  return n;
}

// 32 accumulator columns of this thread's row, + bias, as fp32.
__device__ __forceinline__ void acc_chunk(uint32_t taddr, const float* __restrict__ bias,
                                          float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32_sync(taddr, r);
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 b = __ldg(reinterpret_cast<const float4*>(bias + i));
    v[i] = __uint_as_float(r[i]) + b.x;
    v[i + 1] = __uint_as_float(r[i + 1]) + b.y;
    v[i + 2] = __uint_as_float(r[i + 2]) + b.z;
    v[i + 3] = __uint_as_float(r[i + 3]) + b.w;
  }
}

// q, k, v epilogue for one row and this warp's 128 columns (128 / D heads).
// Every lane runs the epilogue (the TMEM loads are warp-collective); `store`
// says whether this lane's row belongs to the tile and to the pass's
// modality m. t is a valid token index for the loads either way.
template <int D>
struct EpiQkv {
  __device__ __forceinline__ static void run(const GemmParams& p, uint32_t tacc, int t, int s, int m,
                                             int col0, bool store) {
    (void)s;
    const int part = col0 / p.C;  // 0 q, 1 k, 2 v
    const float* bias = p.bias + static_cast<size_t>(m) * p.n_out + col0;
#pragma unroll 1
    for (int hh = 0; hh < 128 / D; ++hh) {
      const int cc = col0 + hh * D;           // first column of this head
      const int head = (cc % p.C) / D;
      const uint32_t ta = tacc + hh * D;
      const float* bh = bias + hh * D;
      __nv_bfloat16* dst = (part == 0 ? p.q_hat : part == 1 ? p.k_hat : p.v) +
                           (static_cast<size_t>(t) * p.heads + head) * D;
      if (part == 2) {
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float v[32];
          acc_chunk(ta + c, bh + c, v);
          uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = v[8 * q4 + e];
            if (store) o[q4] = pack8(y);
          }
        }
        continue;
      }
      // RMSNorm over the head's D values: sum of squares first (TMEM is
      // read twice rather than holding the row in registers)
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float v[32];
        acc_chunk(ta + c, bh + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float r = rsqrtf(ss / D + p.eps);
      const float* g = p.gammas[2 * part + m];
      const float2* rope = p.rope + static_cast<size_t>(t) * (D / 2);
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float v[32];
        acc_chunk(ta + c, bh + c, v);
        uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int i = 8 * q4 + e;
            const float a = v[i] * r * __ldg(g + c + i), b = v[i + 1] * r * __ldg(g + c + i + 1);
            const float2 cs = __ldg(rope + (c + i) / 2);
            y[e] = a * cs.x - b * cs.y;
            y[e + 1] = a * cs.y + b * cs.x;
          }
          if (store) o[q4] = pack8(y);
        }
      }
    }
  }
};

// h_out = h + gate[s, m] * (acc + b_o[m]) for this warp's 128 columns.
struct EpiOut {
  __device__ __forceinline__ static void run(const GemmParams& p, uint32_t tacc, int t, int s, int m,
                                             int col0, bool store) {
    const float* bias = p.bias + static_cast<size_t>(m) * p.n_out + col0;
    const float* gate = p.gate + (static_cast<size_t>(s) * 2 + m) * p.C + col0;
    const uint4* hr = reinterpret_cast<const uint4*>(p.h + static_cast<size_t>(t) * p.C + col0);
    uint4* o = reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(t) * p.C + col0);
#pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
      float v[32];
      acc_chunk(tacc + c, bias + c, v);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float hv[8], y[8];
        unpack8(__ldg(hr + (c / 8) + q4), hv);
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gate + c + 8 * q4));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gate + c + 8 * q4 + 4));
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = fmaf(gv[e], v[8 * q4 + e], hv[e]);
        if (store) o[(c / 8) + q4] = pack8(y);
      }
    }
  }
};

template <class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ GemmCtl ctl;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                                  // kGemmStages x 16 KB
  uint8_t* sB = smem + kGemmStages * kGemmABytes;      // kGemmStages x 32 KB
  volatile int32_t* abort_flag = &ctl.abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int stride = static_cast<int>(gridDim.x);
  const int n_items = p.n_mtiles * p.n_ntiles;
  const int kb_n = p.k / kGemmK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.acc_full[b], 1);
      mbar_init(&ctl.acc_empty[b], 8);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == kGemmProducerWarp && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == kGemmMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == kGemmProducerWarp) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += stride) {
        int mods[2];
        const int np = gemm_passes(p, it, mods);
        const int m0 = (it / p.n_ntiles) * kGemmM, n0 = (it % p.n_ntiles) * kGemmN;
        for (int ps = 0; ps < np && ok; ++ps)
          for (int kb = 0; kb < kb_n; ++kb, ++g) {
            const int st = g % kGemmStages;
            if (!wait_bar(&ctl.empty[st], ((g / kGemmStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&ctl.full[st], kGemmABytes + kGemmBBytes);
            tma_load_2d(sA + st * kGemmABytes, &tmap_a, &ctl.full[st], kb * kGemmK, m0);
            tma_load_2d(sB + st * kGemmBBytes, &tmap_b, &ctl.full[st], kb * kGemmK,
                        mods[ps] * p.n_out + n0);
          }
      }
      if (!ok)
        for (int i = g - kGemmStages > 0 ? g - kGemmStages : 0; i < g; ++i)
          wait_slow(&ctl.full[i % kGemmStages], (i / kGemmStages) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == kGemmMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(kGemmM, kGemmN, 0, 0);
      const uint64_t a_desc0 = smem_desc_sw128(smem_addr(sA), 16, 1024);
      const uint64_t b_desc0 = smem_desc_sw128(smem_addr(sB), 16, 1024);
      int total = 0;
      for (int it = blockIdx.x; it < n_items; it += stride) {
        int mods[2];
        total += gemm_passes(p, it, mods) * kb_n;
      }
      int g = 0, acc = 0;  // stage loads consumed, accumulators filled
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += stride) {
        int mods[2];
        const int np = gemm_passes(p, it, mods);
        for (int ps = 0; ps < np && ok; ++ps, ++acc) {
          const int b = acc & 1;
          // the epilogue has emptied this accumulator (two fills ago)
          if (!wait_bar(&ctl.acc_empty[b], ((acc >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          for (int kb = 0; kb < kb_n; ++kb, ++g) {
            const int st = g % kGemmStages;
            if (!wait_bar(&ctl.full[st], (g / kGemmStages) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
            const uint64_t ad = a_desc0 + static_cast<uint64_t>((st * kGemmABytes) >> 4);
            const uint64_t bd = b_desc0 + static_cast<uint64_t>((st * kGemmBBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kGemmK / 16; ++kk)
              mma_ss(tmem + b * kGemmN, ad + (kk * 32 >> 4), bd + (kk * 32 >> 4), kIdesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
            if (g + kGemmStages < total) mma_commit(&ctl.empty[st]);
          }
          if (!ok) break;
          mma_commit(&ctl.acc_full[b]);
        }
      }
      if (!ok) {
        mma_commit(&ctl.drain);
        wait_slow(&ctl.drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue ---
    const int g4 = warp & 3, h = warp >> 2;  // TMEM lane quarter, 128-column half
    const int row = g4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(g4 * 32) << 16;
    int acc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += stride) {
      int mods[2];
      const int np = gemm_passes(p, it, mods);
      const int t_raw = (it / p.n_ntiles) * kGemmM + row;
      const bool in = t_raw < p.rows;
      const int t = in ? t_raw : p.rows - 1;
      const int col0 = (it % p.n_ntiles) * kGemmN + 128 * h;
      int s = 0, m = 0;
      token_sample_mod(p.cu_seqlens, p.segs, p.n_samples, t, s, m);
      for (int ps = 0; ps < np && ok; ++ps, ++acc) {
        const int b = acc & 1;
        if (!warp_wait_bar(&ctl.acc_full[b], (acc >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        if (col0 < p.n_out)  // uniform across the warp
          Epi::run(p, tmem + lane_off + b * kGemmN + 128 * h, t, s, mods[ps], col0,
                   in && m == mods[ps]);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.acc_empty[b]);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kGemmMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mf
