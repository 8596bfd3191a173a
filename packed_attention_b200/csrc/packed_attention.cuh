// Stage 2: block-diagonal (per-sample) softmax attention on the 5th-generation
// tensor cores.
//
// [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": joint
//  self-attention over packed variable-length samples with per-sample
//  cumulative offsets. The pages run it with FlashAttention's var-len
//  kernels; this kernel is its own design for sm_100a.]
//
// One CTA computes one work item: 128 query rows of one head of one sample,
// attending over the sample's L keys in steps of 128.
//
//   warp 4 (one lane)  TMA producer: the Q tile once, then K_j and V_j tiles
//                      into a ring of NS shared-memory stages (128-byte
//                      swizzled boxes of 128 rows x 64 dims).
//   warp 5 (one lane)  MMA issuer: S_j = Q K_j^T (both operands in shared
//                      memory, fp32 accumulator in TMEM, two S buffers), and
//                      O += P_j V_j (P from TMEM, V from shared memory, O in
//                      TMEM). Completion is signalled with tcgen05.commit.
//                      Warp 5 also owns the TMEM allocation.
//   warps 0-3          softmax, one thread per query row: load the S row from
//                      TMEM, mask keys past the sample end, online max and
//                      sum in the exp2 domain, write P (bf16) to TMEM, and
//                      rescale O in TMEM only when the running max grew by
//                      more than 2^8 (otherwise keep the stale max: p <= 256
//                      stays exact enough in bf16 and cannot overflow fp32).
//                      At the end they normalise O by the row sum and store
//                      bf16 rows, skipping rows past the sample end.
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), O [256,256+d),
// P0 [384,448), P1 [448,512) -- P holds 128 bf16 per row, two per column.
//
// Order of tensor-core work: S0, S1, PV0, S2, PV1, S3, ... S_{j+1} is issued
// before waiting for P_j, so the tensor core computes the next scores while
// the softmax threads work on the current ones. A commit tracks every earlier
// tcgen05 operation of the issuing thread, so when S_j's commit fires PV_{j-2}
// is also complete and the P buffer (j mod 2) may be overwritten.
//
// Every wait is bounded (kWaitLimitNs). A wait that runs out records
// MF_ERR_TIMEOUT in the device error word, raises the CTA's abort flag, and
// every role then leaves its loop, waits (bounded) for its own copies and
// MMAs in flight, and the TMEM is released before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "sm100_ptx.cuh"

namespace mf {

__device__ int32_t g_device_error;

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr int kAttnThreads = 192;
constexpr int kBlockM = MF_TILE_M;
constexpr int kBlockN = MF_TILE_N;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16 (128 bytes, one swizzle span)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct AttnConfig {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBlockM * D * 2;
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kSmemBytes = kTileBytes * (1 + kStages) + 1024;
};

struct AttnParams {
  const mf_segment* segs;
  const mf_work_item* work;
  __nv_bfloat16* out;
  int heads;
  float scale_log2;  // softmax scale * log2(e)
};

struct SharedCtl {
  uint64_t q_full;
  uint64_t kv_full[4];
  uint64_t kv_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
};

__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag,
                                       uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      if (abort_flag) {
        *abort_flag = 1;
        atomicCAS(&g_device_error, 0, static_cast<int32_t>(MF_ERR_TIMEOUT));
      }
      return false;
    }
  }
}

// Bounded wait for the phase of `bar` with the given parity.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, kWaitLimitNs);
}

// Warp-uniform version: the warp continues only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity,
                                              volatile int32_t* abort_flag) {
  const bool ok = wait_bar(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// One 128-column TMEM row per thread (32 lanes per warp), waited.
__device__ __forceinline__ void tmem_ld128_wait(uint32_t taddr, float (&v)[128]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t r[64];
    tmem_ld64_sync(taddr + 64 * c, r);
#pragma unroll
    for (int i = 0; i < 64; ++i) v[64 * c + i] = __uint_as_float(r[i]);
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    packed_attention_kernel(const __grid_constant__ CUtensorMap tmap_q,
                            const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  using Cfg = AttnConfig<D>;
  constexpr int NS = Cfg::kStages;
  constexpr int kTile = Cfg::kTileBytes;

  extern __shared__ uint8_t smem_raw[];
  __shared__ SharedCtl ctl;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kTile;
  volatile int32_t* abort_flag = &ctl.abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const mf_work_item wi = p.work[blockIdx.x];
  const mf_segment seg = p.segs[wi.seg];
  const int q0 = seg.start + wi.q_tile * kBlockM;
  const int seg_end = seg.start + seg.len;
  const int n_kv = (seg.len + kBlockN - 1) / kBlockN;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.s_full[b], 1);
      mbar_init(&ctl.p_full[b], 4);
    }
    mbar_init(&ctl.pv_done, 1);
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == 5) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer ---
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(&ctl.q_full, kTile);
#pragma unroll
      for (int b = 0; b < Cfg::kBoxes; ++b)
        tma_load_3d(sQ + b * kBoxBytes, &tmap_q, &ctl.q_full, 64 * b, wi.head, q0);
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int which = 0; which < 2; ++which) {
          const int i = 2 * j + which;
          const int st = i % NS;
          if (!wait_bar(&ctl.kv_empty[st], ((i / NS) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl.kv_full[st], kTile);
          const CUtensorMap* map = which ? &tmap_v : &tmap_k;
#pragma unroll
          for (int b = 0; b < Cfg::kBoxes; ++b)
            tma_load_3d(sKV + st * kTile + b * kBoxBytes, map, &ctl.kv_full[st], 64 * b, wi.head,
                        seg.start + j * kBlockN);
          issued = i + 1;
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA can exit.
        wait_slow(&ctl.q_full, 0, nullptr, 100000000ull);
        for (int i = issued - NS > 0 ? issued - NS : 0; i < issued; ++i)
          wait_slow(&ctl.kv_full[i % NS], (i / NS) & 1, nullptr, 100000000ull);
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------- MMA issuer ---
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlockM, D, 0, 1);
      const uint32_t q_addr = smem_addr(sQ);
      const uint32_t kv_addr = smem_addr(sKV);
      const int total_loads = 2 * n_kv;
      bool ok = wait_bar(&ctl.q_full, 0, abort_flag);
      tc_fence_after_sync();

      // S_jj = Q K_jj^T into S buffer (jj mod 2).
      auto issue_s = [&](int jj) -> bool {
        const int i = 2 * jj;
        const int st = i % NS;
        if (!wait_bar(&ctl.kv_full[st], (i / NS) & 1, abort_flag)) return false;
        tc_fence_after_sync();
        const uint32_t k_addr = kv_addr + st * kTile;
        const uint32_t d_tmem = tmem + ((jj & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kBoxBytes + (kk % 4) * 32;
          mma_ss(d_tmem, smem_desc_sw128(q_addr + off, 16, 1024),
                 smem_desc_sw128(k_addr + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
        }
        if (i + NS < total_loads) mma_commit(&ctl.kv_empty[st]);
        mma_commit(&ctl.s_full[jj & 1]);
        return true;
      };

      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) { ok = false; break; }
        if (!wait_bar(&ctl.p_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const int i = 2 * j + 1;
        const int st = i % NS;
        if (!wait_bar(&ctl.kv_full[st], (i / NS) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const uint32_t v_addr = kv_addr + st * kTile;
        const uint32_t p_tmem = tmem + ((j & 1) ? kColP1 : kColP0);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // V is [keys, d] with d contiguous: an MN-major B operand. 16 keys per
          // step = two 8-row swizzle atoms (2 KB); d blocks of 64 are a box apart.
          mma_ts(tmem + kColO, p_tmem + kk * 8, smem_desc_sw128(v_addr + kk * 2048, kBoxBytes, 1024),
                 kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (i + NS < total_loads) mma_commit(&ctl.kv_empty[st]);
        mma_commit(&ctl.pv_done);
      }
      if (!ok) {
        // Every MMA issued so far must finish before TMEM is released.
        mma_commit(&ctl.drain);
        wait_slow(&ctl.drain, 0, nullptr, 100000000ull);
      }
    }
  } else {
    // ----------------------------------------------------------- softmax ---
    const int row = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running max of s * scale * log2(e)
    float l = 0.0f;       // running sum of p
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!warp_wait_bar(&ctl.s_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after_sync();
      float s[128];
      tmem_ld128_wait(tmem + lane_off + ((j & 1) ? kColS1 : kColS0), s);
      const int valid = seg.len - j * kBlockN;  // keys of this step inside the sample
      if (valid < kBlockN) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const float m_new = fmaxf(m, m_tile);
      // pv_done must be observed once per phase, in order (a parity wait cannot
      // tell phase j-1 from phase j-3): PV_{j-1} is waited for here when O has
      // to be rescaled, otherwise just before P_j is handed to the MMA warp.
      bool pv_prev_seen = (j == 0);
      if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
        const float factor = ex2_approx(m - m_new);  // 0 on the first step
        l *= factor;
        if (j > 0) {
          // O holds PV_0..PV_{j-1}: wait for the last one, then scale the row.
          if (!warp_wait_bar(&ctl.pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
          pv_prev_seen = true;
          tc_fence_after_sync();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            const uint32_t ta = tmem + lane_off + kColO + 32 * c;
            tmem_ld32_sync(ta, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
            tmem_st32_sync(ta, r);
          }
        }
        m = m_new;
      }
      float l0 = 0.f, l1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(s[2 * c], sl2, -m));
        const float p1 = ex2_approx(fmaf(s[2 * c + 1], sl2, -m));
        l0 += p0;
        l1 += p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l += l0 + l1;
      tmem_st64_sync(tmem + lane_off + ((j & 1) ? kColP1 : kColP0), pk);
      if (!pv_prev_seen && !warp_wait_bar(&ctl.pv_done, (j - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.p_full[j & 1]);
    }
    if (ok && warp_wait_bar(&ctl.pv_done, (n_kv - 1) & 1, abort_flag)) {
      tc_fence_after_sync();
      const int q_row = q0 + row;
      const float inv_l = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(q_row) * p.heads + wi.head) * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32_sync(tmem + lane_off + kColO + 32 * c, r);
        if (q_row < seg_end) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(r[8 * v4 + 0]) * inv_l, __uint_as_float(r[8 * v4 + 1]) * inv_l);
            o.y = pack_bf16x2(__uint_as_float(r[8 * v4 + 2]) * inv_l, __uint_as_float(r[8 * v4 + 3]) * inv_l);
            o.z = pack_bf16x2(__uint_as_float(r[8 * v4 + 4]) * inv_l, __uint_as_float(r[8 * v4 + 5]) * inv_l);
            o.w = pack_bf16x2(__uint_as_float(r[8 * v4 + 6]) * inv_l, __uint_as_float(r[8 * v4 + 7]) * inv_l);
            dst[4 * c + v4] = o;
          }
        }
      }
    }
  }

  // ---------------------------------------------------------- teardown ---
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mf
