// Backward of the packed joint attention, for training.
//
// [Mage-Flow video overview, 00:05:08, and paper summary, "Training
//  Infrastructure": the fused-kernel speedup is a training speedup. The
//  backward here is the chain rule through the forward of this library.]
//
// With dO = dL/dout, the forward's bf16 output `out` and its per-row natural
// log-normaliser lse (written by the forward), for query t and key u of one
// sample and head, s_tu = scale * q_hat_t . k_hat_u:
//   D_t       = dO_t . out_t                                   bwd_delta_kernel
//   P_tu      = exp(s_tu - lse_t)                              (recomputed)
//   dS_tu     = P_tu * (dO_t . v_u - D_t)
//   dv_u      = sum_t P_tu dO_t                                attn_bwd_dkdv_kernel
//   dk_hat_u  = scale * sum_t dS_tu q_hat_t                    attn_bwd_dkdv_kernel
//   dq_hat_t  = scale * sum_u dS_tu k_hat_u                    attn_bwd_dq_kernel
// then back through the rotation (transposed) and the RMSNorm, with the four
// gamma gradients summed over tokens and heads    qk_prologue_bwd_kernel,
//                                                  dgamma_reduce_kernel
//
// The two attention kernels are persistent tcgen05 kernels built like the
// forward: TMA loads into 128-byte-swizzled shared tiles, MMAs issued by one
// thread with fp32 accumulators in TMEM, eight softmax warps (a TMEM lane
// quarter each, two warps per quarter splitting the 128 columns), bounded
// mbarrier waits throughout. A work item of the forward's list (256 rows of
// one head of one sample) is done as two passes of 128 rows.
//
// Operands reused across a pass sit in TMEM where there is room, and so do P
// and dS: an MMA with A in TMEM reads one operand (4 KB for 128 x 128 x 16)
// from shared memory instead of two.
//
// dK/dV kernel, per pass: 128 key rows; K_hat and V stay in shared memory and
// every query step j brings Q_hat_j and dO_j (2-stage rings each). The
// per-query statistics of a step (-lse in log2 units, D) go through a small
// per-warp shared array and are read as broadcast pairs (measured faster than
// warp shuffles).
// TMEM columns:
//   S^T = K_hat Q_hat_j^T [0,128)   P^T (bf16) over [0,32) and [64,96)
//   dP^T = V dO_j^T     [128,256)   dS^T (bf16) over [128,160) and [192,224)
//   dV accumulator      [256,256+d)
//   dK accumulator      [384,384+d)
// P^T and dS^T are the TMEM A operands of dV += P^T dO_j and dK += dS^T Q_j.
// MMA order per step: dV_j, S^T_{j+1}, dK_j, dP^T_{j+1}: the exponentials of
// step j+1 overlap dK_j and dP^T_{j+1}, its dS overlaps dV_{j+1} and
// S^T_{j+2}. MMAs of one thread execute in issue order, so S^T_{j+1}
// overwrites P^T_j only after dV_j has read it (and dP^T_{j+1} dS^T_j only
// after dK_j).
//
// dQ kernel, per pass: 128 query rows. Q_hat and dO are read once per pass
// into TMEM (the A operands of S and dP); every key step brings K_hat_j
// (4-stage ring) and V_j (3-stage ring). TMEM: S [0,128), dP [128,256) with
// dS (bf16) over [128,160) and [192,224), dQ accumulator [256,256+d), Q_hat
// [384,384+d/2), dO [448,448+d/2). Per step: S_{j+1} as soon as every
// softmax warp holds S_j in registers, dQ_j once dS_j is written, dP_{j+1}.
#pragma once

#include "packed_attention.cuh"

namespace mf {

// Warps 0-7 softmax and epilogue, 8 TMA producer, 9 MMA issuer. Ten warps
// put three on two of the SM's four sub-partitions, which caps a thread at
// 168 registers.
constexpr int kBwdThreads = 320;
constexpr int kBwdProducerWarp = 8;
constexpr int kBwdMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;

// kFix: tiles kept in shared memory for a whole pass (K_hat, V in dK/dV; the
// dQ kernel keeps Q_hat and dO in TMEM instead). kRingX: the ring operand
// held longest (Q_hat in dK/dV, K_hat in dQ); kRingY: the one released after
// its first MMA (dO in dK/dV, V in dQ).
template <int D, bool kDq>
struct BwdConfig {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kSubM * D * 2;
  static constexpr int kFix = kDq ? 0 : 2;
  static constexpr int kRingX = kDq ? 4 : 2;
  static constexpr int kRingY = 2;
  // 2 KB per softmax warp to stage its output rows.
  static constexpr int kStageBytes = 8 * 2048;
  static constexpr int kSmemBytes = kTileBytes * (kFix + kRingX + kRingY) + kStageBytes + 1024;
};

// 32 rows x 64 bytes of one warp (lane = row) go to rows gbase + r * stride,
// r < valid_rows, through the warp's 2 KB of shared memory: stage_put places
// the lane's 16-byte piece c, stage_flush stores, and each of its store
// instructions writes eight whole 64-byte row segments instead of 32
// scattered 16-byte pieces. Piece c of row r sits at c ^ ((r / 2) % 4), so
// that neither side has bank conflicts.
// (stage is a shared-memory address.)
__device__ __forceinline__ void stage_put(uint32_t stage, int lane, int c, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                   stage + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// (buf, buf_bytes: the destination buffer, for the checked build's range check.)
__device__ __forceinline__ void stage_flush(uint32_t stage, int lane, uint8_t* gbase, size_t stride,
                                            int valid_rows, const void* buf, size_t buf_bytes) {
  __syncwarp();
  const int q = lane & 3;
#pragma unroll 1
  for (int i = 0; i < 4; ++i) {
    const int rr = 8 * i + (lane >> 2);
    uint4 o;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
                 : "r"(stage + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4))
                 : "memory");
    uint8_t* dst = gbase + rr * stride + q * 16;
    if (rr < valid_rows && in_span(dst, 16, buf, buf_bytes)) *reinterpret_cast<uint4*>(dst) = o;
  }
  __syncwarp();
}

struct BwdParams {
  const mf_segment* segs;
  const mf_work_item* work;
  int n_segs;
  const float* lse;       // [heads, total_tokens], natural log
  const float* delta;     // [heads, total_tokens]
  float* dhat;            // fp32 [total_tokens, heads, D]: dk_hat or dq_hat
  __nv_bfloat16* dv;      // bf16 [total_tokens, heads, D] (dK/dV kernel)
  const uint4* q_rows;    // q_hat [total_tokens, heads, D] (dQ kernel: read into TMEM)
  const uint4* do_rows;   // dO, same layout (dQ kernel)
  int n_work;
  int heads;
  int total_tokens;
  float scale;            // softmax scale
  float scale_log2;       // scale * log2(e)
};

struct BwdCtl {
  uint64_t fix_full, fix_empty;
  uint64_t x_full[4], x_empty[4];
  uint64_t y_full[3], y_empty[3];
  uint64_t s_full, s_free, dp_full;
  uint64_t p_ready, ds_ready, q_ready;
  uint64_t acc_ready, acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
};

// D (+)= A (TMEM, bf16: 128 lanes x 128 K, K 0..63 in columns [0,32) and
// K 64..127 in [64,96)) * B (shared, MN-major [K = 128 rows][N = D]).
// Low half of a shared-memory descriptor made by smem_desc_sw128(.., .., 1024),
// whose high half is kDescHiSw128, for issue_qk.
__device__ __forceinline__ uint32_t lo32(uint64_t desc) { return static_cast<uint32_t>(desc); }

template <int D>
__device__ __forceinline__ void issue_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(kSubM, D, 0, 1);
  const uint32_t b_lo = lo32(b_desc);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_lo(d_tmem, a_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
              b_lo + static_cast<uint32_t>(kk * (2048 >> 4)), kIdesc,
              (accumulate || kk > 0) ? 1u : 0u);
}

template <int D, bool kDq>
__device__ __forceinline__ void bwd_init(BwdCtl& ctl, int warp) {
  if (threadIdx.x == 0) {
    mbar_init(&ctl.fix_full, 1);
    mbar_init(&ctl.fix_empty, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&ctl.x_full[s], 1);
      mbar_init(&ctl.x_empty[s], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&ctl.y_full[s], 1);
      mbar_init(&ctl.y_empty[s], 1);
    }
    mbar_init(&ctl.s_full, 1);
    mbar_init(&ctl.s_free, 8);
    mbar_init(&ctl.dp_full, 1);
    mbar_init(&ctl.p_ready, 8);
    mbar_init(&ctl.ds_ready, 8);
    mbar_init(&ctl.q_ready, 8);
    mbar_init(&ctl.acc_ready, 1);
    mbar_init(&ctl.acc_empty, 8);
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
}

__device__ __forceinline__ void bwd_teardown(uint32_t tmem, int warp) {
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Producer for both kernels: per pass, the two fixed tiles (rows r0 of
// fix_a / fix_b), then per step j the ring tiles (rows seg_start + 128 j of
// ring_x / ring_y).
template <int D, bool kDq>
__device__ __forceinline__ void bwd_producer(const BwdParams& p, BwdCtl& ctl, uint8_t* sFix,
                                             uint8_t* sX, uint8_t* sY, const CUtensorMap* fix_a,
                                             const CUtensorMap* fix_b, const CUtensorMap* ring_x,
                                             const CUtensorMap* ring_y,
                                             volatile int32_t* abort_flag) {
  using Cfg = BwdConfig<D, kDq>;
  constexpr int NX = Cfg::kRingX, NY = Cfg::kRingY, kTile = Cfg::kTileBytes;
  const int stride = static_cast<int>(gridDim.x);
  int pc = 0, gx = 0, gy = 0;
  bool ok = true;
  for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
    const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
    // Tiles start inside the tensor (rows past T read as zeros).
    if (kChecked) {
      in_bounds(it.head, p.heads);
      in_bounds(it.q0, p.total_tokens);
      in_bounds(it.seg_start + it.seg_len - 1, p.total_tokens);
    }
    const int passes = it.b_valid ? 2 : 1;
    for (int t = 0; t < passes && ok; ++t) {
      const int r0 = it.q0 + t * kSubM;
      if (Cfg::kFix > 0) {
        if (!wait_bar(&ctl.fix_empty, (pc & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&ctl.fix_full, 2 * kTile);
#pragma unroll
        for (int b = 0; b < Cfg::kBoxes; ++b) {
          tma_load_3d(sFix + b * kBoxBytes, fix_a, &ctl.fix_full, 64 * b, it.head, r0);
          tma_load_3d(sFix + kTile + b * kBoxBytes, fix_b, &ctl.fix_full, 64 * b, it.head, r0);
        }
        ++pc;
      }
      for (int j = 0; j < it.n_kv && ok; ++j) {
        const int c = it.seg_start + j * kBlockN;
        {
          const int st = gx % NX;
          if (!wait_bar(&ctl.x_empty[st], ((gx / NX) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&ctl.x_full[st], kTile);
#pragma unroll
          for (int b = 0; b < Cfg::kBoxes; ++b)
            tma_load_3d(sX + st * kTile + b * kBoxBytes, ring_x, &ctl.x_full[st], 64 * b, it.head, c);
          ++gx;
        }
        {
          const int st = gy % NY;
          if (!wait_bar(&ctl.y_empty[st], ((gy / NY) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&ctl.y_full[st], kTile);
#pragma unroll
          for (int b = 0; b < Cfg::kBoxes; ++b)
            tma_load_3d(sY + st * kTile + b * kBoxBytes, ring_y, &ctl.y_full[st], 64 * b, it.head, c);
          ++gy;
        }
      }
    }
  }
  if (!ok) {
    // Let every copy already issued land before the CTA can exit.
    if (pc > 0) wait_slow(&ctl.fix_full, (pc - 1) & 1, nullptr, kDrainLimitNs);
    for (int i = gx - NX > 0 ? gx - NX : 0; i < gx; ++i)
      wait_slow(&ctl.x_full[i % NX], (i / NX) & 1, nullptr, kDrainLimitNs);
    for (int i = gy - NY > 0 ? gy - NY : 0; i < gy; ++i)
      wait_slow(&ctl.y_full[i % NY], (i / NY) & 1, nullptr, kDrainLimitNs);
  }
}

// Passes and steps this CTA will run (for releasing only refilled slots).
__device__ __forceinline__ void bwd_counts(const BwdParams& p, int& passes, int& steps) {
  passes = steps = 0;
  const int stride = static_cast<int>(gridDim.x);
  for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
    const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
    const int np = it.b_valid ? 2 : 1;
    passes += np;
    steps += np * it.n_kv;
  }
}

// ---------------------------------------------------------------- dK, dV ---

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_do, const BwdParams p) {
  using Cfg = BwdConfig<D, false>;
  constexpr int NX = Cfg::kRingX, NY = Cfg::kRingY, kTile = Cfg::kTileBytes;
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdCtl ctl;
  __shared__ __align__(16) float s_stat[8][2][64];  // per softmax warp: -lse2, D of 64 queries
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;              // fixed: K_hat then V
  uint8_t* sV = smem + kTile;
  uint8_t* sX = smem + 2 * kTile;  // ring of Q_hat
  uint8_t* sY = sX + NX * kTile;   // ring of dO
  uint8_t* sStage = sY + NY * kTile;  // 2 KB per softmax warp
  volatile int32_t* abort_flag = &ctl.abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (warp == kBwdProducerWarp && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
    prefetch_tmap(&tmap_do);
  }
  bwd_init<D, false>(ctl, warp);
  const uint32_t tmem = ctl.tmem_base;
  const int stride = static_cast<int>(gridDim.x);

  if (warp == kBwdProducerWarp) {
    if (lane == 0)
      bwd_producer<D, false>(p, ctl, sK, sX, sY, &tmap_k, &tmap_v, &tmap_q, &tmap_do, abort_flag);
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0) {
      const uint64_t k_desc = smem_desc_sw128(smem_addr(sK), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_addr(sV), 16, 1024);
      const uint64_t x_k = smem_desc_sw128(smem_addr(sX), 16, 1024);          // Q_hat as B of S^T
      const uint64_t x_mn = smem_desc_sw128(smem_addr(sX), kBoxBytes, 1024);  // Q_hat as B of dK
      const uint64_t y_k = smem_desc_sw128(smem_addr(sY), 16, 1024);          // dO as B of dP^T
      const uint64_t y_mn = smem_desc_sw128(smem_addr(sY), kBoxBytes, 1024);  // dO as B of dV
      constexpr uint64_t kStep = static_cast<uint64_t>(kTile >> 4);
      int total_passes, total_steps;
      bwd_counts(p, total_passes, total_steps);
      int pc = 0, g = 0;
      uint32_t nph = 0;
      bool ok = true;
      for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
        const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
        const int passes = it.b_valid ? 2 : 1;
        for (int t = 0; t < passes && ok; ++t) {
          const int n = it.n_kv;
          if (!wait_bar(&ctl.fix_full, pc & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          if (!wait_bar(&ctl.x_full[g % NX], (g / NX) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          issue_qk<D>(tmem + kColS, lo32(k_desc), lo32(x_k + (g % NX) * kStep));
          mma_commit(&ctl.s_full);
          if (!wait_bar(&ctl.y_full[g % NY], (g / NY) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          issue_qk<D>(tmem + kColDP, lo32(v_desc), lo32(y_k + (g % NY) * kStep));
          mma_commit(&ctl.dp_full);
          for (int j = 0; j < n && ok; ++j) {
            const int gj = g + j, gn = gj + 1;
            const bool more = j + 1 < n;
            if (!wait_bar(&ctl.p_ready, nph & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
            if (j == 0 && pc > 0) {
              // the previous pass's accumulators have been read out
              if (!wait_bar(&ctl.acc_empty, (pc - 1) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
            }
            issue_tmem_a<D>(tmem + kColDV, tmem + kColS, y_mn + (gj % NY) * kStep, j > 0);
            if (gj + NY < total_steps) mma_commit(&ctl.y_empty[gj % NY]);
            if (more) {
              if (!wait_bar(&ctl.x_full[gn % NX], (gn / NX) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
              issue_qk<D>(tmem + kColS, lo32(k_desc), lo32(x_k + (gn % NX) * kStep));
              mma_commit(&ctl.s_full);
            }
            if (!wait_bar(&ctl.ds_ready, nph & 1, abort_flag)) { ok = false; break; }
            ++nph;
            tc_fence_after_sync();
            issue_tmem_a<D>(tmem + kColDK, tmem + kColDP, x_mn + (gj % NX) * kStep, j > 0);
            if (gj + NX < total_steps) mma_commit(&ctl.x_empty[gj % NX]);
            if (more) {
              if (!wait_bar(&ctl.y_full[gn % NY], (gn / NY) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
              issue_qk<D>(tmem + kColDP, lo32(v_desc), lo32(y_k + (gn % NY) * kStep));
              mma_commit(&ctl.dp_full);
            }
          }
          if (!ok) break;
          if (pc + 1 < total_passes) mma_commit(&ctl.fix_empty);
          mma_commit(&ctl.acc_ready);
          g += n;
          ++pc;
        }
      }
      if (!ok) {
        mma_commit(&ctl.drain);
        wait_slow(&ctl.drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // ------------------------------------------- softmax and epilogue ---
    const int g4 = warp & 3, h = warp >> 2;  // TMEM lane quarter, column half
    const uint32_t lane_off = static_cast<uint32_t>(g4 * 32) << 16;
    const uint64_t sl2x2 = f32x2(p.scale_log2, p.scale_log2);
    uint32_t ns = 0, nd = 0;
    int pc = 0;
    bool ok = true;
    for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
      const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
      const int passes = it.b_valid ? 2 : 1;
      const int seg_end = it.seg_start + it.seg_len;
      const size_t stat0 = static_cast<size_t>(it.head) * p.total_tokens;
      // -lse (log2 units) and D of query columns 2*lane, 2*lane+1 of this
      // warp's half of step j; queries past the sample end get -lse = -inf
      // (P = 0) and D = 0.
      auto load_stats = [&](int j, float& nl0, float& nl1, float& d0, float& d1) {
        const int q0 = it.seg_start + j * kBlockN + 64 * h + 2 * lane;
        const long long n_stat = static_cast<long long>(p.heads) * p.total_tokens;
        const bool in0 = q0 < seg_end && in_bounds(stat0 + q0, n_stat);
        const bool in1 = q0 + 1 < seg_end && in_bounds(stat0 + q0 + 1, n_stat);
        nl0 = in0 ? -__ldg(p.lse + stat0 + q0) * kLog2e : -INFINITY;
        nl1 = in1 ? -__ldg(p.lse + stat0 + q0 + 1) * kLog2e : -INFINITY;
        d0 = in0 ? __ldg(p.delta + stat0 + q0) : 0.0f;
        d1 = in1 ? __ldg(p.delta + stat0 + q0 + 1) : 0.0f;
      };
      for (int t = 0; t < passes && ok; ++t, ++pc) {
        const int r0 = it.q0 + t * kSubM;
        float nl0, nl1, d0, d1;
        load_stats(0, nl0, nl1, d0, d1);
        for (int j = 0; j < it.n_kv; ++j) {
          // next step's statistics, in flight while this step computes
          float nnl0 = 0.f, nnl1 = 0.f, nd0 = 0.f, nd1 = 0.f;
          if (j + 1 < it.n_kv) load_stats(j + 1, nnl0, nnl1, nd0, nd1);
          float* st_l = s_stat[warp][0];
          float* st_d = s_stat[warp][1];
          __syncwarp();
          st_l[2 * lane] = nl0; st_l[2 * lane + 1] = nl1;
          st_d[2 * lane] = d0; st_d[2 * lane + 1] = d1;
          __syncwarp();
          if (!warp_wait_bar(&ctl.s_full, ns & 1, abort_flag)) { ok = false; break; }
          ++ns;
          tc_fence_after_sync();
          uint64_t pp[32];
          {
            uint32_t sr[64];
            tmem_ld64_sync(tmem + lane_off + kColS + 64 * h, sr);
            uint32_t pk[32];
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
              const float2 nl = reinterpret_cast<const float2*>(st_l)[c2];
              const uint64_t x = fma_f32x2(
                  f32x2(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1])), sl2x2,
                  f32x2(nl.x, nl.y));
              float x0, x1;
              f32x2_split(x, x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              pp[c2] = f32x2(p0, p1);
              pk[c2] = pack_bf16x2(p0, p1);
            }
            // P^T over the first 32 columns of this warp's half of S^T
            tmem_st32_sync(tmem + lane_off + kColS + 64 * h, pk);
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.p_ready);
          if (!warp_wait_bar(&ctl.dp_full, nd & 1, abort_flag)) { ok = false; break; }
          ++nd;
          tc_fence_after_sync();
          {
            uint32_t pk[32];
            // dS in two halves of 32 columns (keeps dP and P in registers together)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t dr[32];
              tmem_ld32_sync(tmem + lane_off + kColDP + 64 * h + 32 * half, dr);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c2 = 16 * half + i;
                const float2 dd = reinterpret_cast<const float2*>(st_d)[c2];
                const uint64_t ds = mul_f32x2(
                    pp[c2], sub_f32x2(f32x2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])),
                                      f32x2(dd.x, dd.y)));
                float a, b;
                f32x2_split(ds, a, b);
                pk[c2] = pack_bf16x2(a, b);
              }
            }
            tmem_st32_sync(tmem + lane_off + kColDP + 64 * h, pk);
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.ds_ready);
          nl0 = nnl0; nl1 = nnl1; d0 = nd0; d1 = nd1;
        }
        if (!ok) break;
        // ---- epilogue: dv (bf16) and dk_hat = scale * acc (fp32) rows ----
        if (!warp_wait_bar(&ctl.acc_ready, pc & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const int tok0 = r0 + g4 * 32;  // token of this warp's first key row
        const int valid_rows = seg_end - tok0;
        const uint32_t stage = smem_addr(sStage) + warp * 2048;
        // bytes of one fp32 [T, H, D] tensor (the bf16 dv is half of it)
        const size_t rows_bytes = static_cast<size_t>(p.total_tokens) * p.heads * D * 4;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          const int col = h * (D / 2) + 32 * c;
          const size_t orow0 = (static_cast<size_t>(tok0) * p.heads + it.head) * D + col;
          uint32_t r[32];
          tmem_ld32_sync(tmem + lane_off + kColDV + col, r);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            stage_put(stage, lane, v4,
                      make_uint4(pack_bf16x2(__uint_as_float(r[8 * v4 + 0]), __uint_as_float(r[8 * v4 + 1])),
                                 pack_bf16x2(__uint_as_float(r[8 * v4 + 2]), __uint_as_float(r[8 * v4 + 3])),
                                 pack_bf16x2(__uint_as_float(r[8 * v4 + 4]), __uint_as_float(r[8 * v4 + 5])),
                                 pack_bf16x2(__uint_as_float(r[8 * v4 + 6]), __uint_as_float(r[8 * v4 + 7]))));
          stage_flush(stage, lane, reinterpret_cast<uint8_t*>(p.dv + orow0),
                      static_cast<size_t>(p.heads) * D * 2, valid_rows, p.dv, rows_bytes / 2);
          tmem_ld32_sync(tmem + lane_off + kColDK + col, r);
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int e = 16 * k2 + 4 * v4;
              stage_put(stage, lane, v4,
                        make_uint4(__float_as_uint(__uint_as_float(r[e + 0]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 1]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 2]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 3]) * p.scale)));
            }
            stage_flush(stage, lane, reinterpret_cast<uint8_t*>(p.dhat + orow0 + 16 * k2),
                        static_cast<size_t>(p.heads) * D * 4, valid_rows, p.dhat, rows_bytes);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.acc_empty);
      }
    }
  }
  bwd_teardown(tmem, warp);
}

// -------------------------------------------------------------------- dQ ---

// D (+)= A (TMEM, bf16 [128 lanes][K = D], D/2 consecutive columns) *
// B^T (shared, K-major [N = 128 rows][K = D]): M = 128, N = 128.
template <int D>
__device__ __forceinline__ void issue_rows_tmem(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(kSubM, kBlockN, 0, 0);
  const uint32_t b_lo = lo32(b_desc);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_ts_lo(d_tmem, a_tmem + kk * 8,
              b_lo + static_cast<uint32_t>(((kk / 4) * kBoxBytes + (kk % 4) * 32) >> 4), kIdesc,
              kk > 0 ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v,
                       const __grid_constant__ CUtensorMap tmap_do, const BwdParams p) {
  using Cfg = BwdConfig<D, true>;
  constexpr int NX = Cfg::kRingX, NY = Cfg::kRingY, kTile = Cfg::kTileBytes;
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColQ = 384, kColO = 448;

  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdCtl ctl;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem;              // ring of K_hat
  uint8_t* sY = sX + NX * kTile;   // ring of V
  uint8_t* sStage = sY + NY * kTile;  // 2 KB per softmax warp
  volatile int32_t* abort_flag = &ctl.abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  (void)tmap_q;
  (void)tmap_do;

  if (warp == kBwdProducerWarp && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  bwd_init<D, true>(ctl, warp);
  const uint32_t tmem = ctl.tmem_base;
  const int stride = static_cast<int>(gridDim.x);

  if (warp == kBwdProducerWarp) {
    if (lane == 0)
      bwd_producer<D, true>(p, ctl, nullptr, sX, sY, nullptr, nullptr, &tmap_k, &tmap_v, abort_flag);
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0) {
      const uint64_t x_k = smem_desc_sw128(smem_addr(sX), 16, 1024);          // K_hat as B of S
      const uint64_t x_mn = smem_desc_sw128(smem_addr(sX), kBoxBytes, 1024);  // K_hat as B of dQ
      const uint64_t y_k = smem_desc_sw128(smem_addr(sY), 16, 1024);          // V as B of dP
      constexpr uint64_t kStep = static_cast<uint64_t>(kTile >> 4);
      int total_passes, total_steps;
      bwd_counts(p, total_passes, total_steps);
      int pc = 0, g = 0;
      uint32_t nph = 0, nsf = 0;
      bool ok = true;
      for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
        const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
        const int passes = it.b_valid ? 2 : 1;
        for (int t = 0; t < passes && ok; ++t) {
          const int n = it.n_kv;
          // Q_hat and dO of the pass are in TMEM (the previous pass's MMAs
          // had completed before the softmax warps wrote them)
          if (!wait_bar(&ctl.q_ready, pc & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          if (!wait_bar(&ctl.x_full[g % NX], (g / NX) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          issue_rows_tmem<D>(tmem + kColS, tmem + kColQ, x_k + (g % NX) * kStep);
          mma_commit(&ctl.s_full);
          if (!wait_bar(&ctl.y_full[g % NY], (g / NY) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          issue_rows_tmem<D>(tmem + kColDP, tmem + kColO, y_k + (g % NY) * kStep);
          mma_commit(&ctl.dp_full);
          if (g + NY < total_steps) mma_commit(&ctl.y_empty[g % NY]);
          for (int j = 0; j < n && ok; ++j) {
            const int gj = g + j, gn = gj + 1;
            const bool more = j + 1 < n;
            if (more) {
              // S_{j+1} as soon as every softmax warp holds S_j
              if (!wait_bar(&ctl.s_free, nsf & 1, abort_flag)) { ok = false; break; }
              ++nsf;
              if (!wait_bar(&ctl.x_full[gn % NX], (gn / NX) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
              issue_rows_tmem<D>(tmem + kColS, tmem + kColQ, x_k + (gn % NX) * kStep);
              mma_commit(&ctl.s_full);
            }
            if (!wait_bar(&ctl.ds_ready, nph & 1, abort_flag)) { ok = false; break; }
            ++nph;
            tc_fence_after_sync();
            issue_tmem_a<D>(tmem + kColDQ, tmem + kColDP, x_mn + (gj % NX) * kStep, j > 0);
            if (gj + NX < total_steps) mma_commit(&ctl.x_empty[gj % NX]);
            if (more) {
              // dP_{j+1} overwrites dS_j only after dQ_j (issued above) has read it
              if (!wait_bar(&ctl.y_full[gn % NY], (gn / NY) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
              issue_rows_tmem<D>(tmem + kColDP, tmem + kColO, y_k + (gn % NY) * kStep);
              mma_commit(&ctl.dp_full);
              if (gn + NY < total_steps) mma_commit(&ctl.y_empty[gn % NY]);
            }
          }
          if (!ok) break;
          // the last S_j was loaded too: consume its s_free phase
          if (!wait_bar(&ctl.s_free, nsf & 1, abort_flag)) { ok = false; break; }
          ++nsf;
          mma_commit(&ctl.acc_ready);
          g += n;
          ++pc;
        }
      }
      if (!ok) {
        mma_commit(&ctl.drain);
        wait_slow(&ctl.drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // ------------------------------------------- softmax and epilogue ---
    const int g4 = warp & 3, h = warp >> 2;
    const int row = g4 * 32 + lane;  // query row of the pass
    const uint32_t lane_off = static_cast<uint32_t>(g4 * 32) << 16;
    const uint64_t sl2x2 = f32x2(p.scale_log2, p.scale_log2);
    uint32_t ns = 0, nd = 0;
    int pc = 0;
    bool ok = true;
    for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
       idx = next_item(p.work, p.n_work, idx + stride, stride)) {
      const ItemInfo it = load_item(p.segs, p.n_segs, p.work, idx);
      const int passes = it.b_valid ? 2 : 1;
      const int seg_end = it.seg_start + it.seg_len;
      for (int t = 0; t < passes && ok; ++t, ++pc) {
        const int r0 = it.q0 + t * kSubM;
        const int q = r0 + row;
        const bool row_in = q < seg_end;
        // This warp's half of the row's Q_hat and dO into TMEM (columns
        // [kColQ + D/4 * h, +D/4) and the same for dO); rows past the pack
        // are zeros. The previous pass's MMAs completed before its epilogue.
        {
          constexpr int kV = D / 16;  // 16-byte vectors per half row
          const size_t base = (static_cast<size_t>(q) * p.heads + it.head) * (D / 8) + kV * h;
          uint32_t qv[D / 4], ov[D / 4];
#pragma unroll
          for (int v = 0; v < kV; ++v) {
            const bool in = q < p.total_tokens &&
                            in_bounds(base + v, static_cast<long long>(p.total_tokens) * p.heads * (D / 8));
            const uint4 a = in ? __ldg(p.q_rows + base + v) : make_uint4(0, 0, 0, 0);
            const uint4 b = in ? __ldg(p.do_rows + base + v) : make_uint4(0, 0, 0, 0);
            qv[4 * v] = a.x; qv[4 * v + 1] = a.y; qv[4 * v + 2] = a.z; qv[4 * v + 3] = a.w;
            ov[4 * v] = b.x; ov[4 * v + 1] = b.y; ov[4 * v + 2] = b.z; ov[4 * v + 3] = b.w;
          }
          if constexpr (D == 128) {
            tmem_st32_sync(tmem + lane_off + kColQ + 32 * h, qv);
            tmem_st32_sync(tmem + lane_off + kColO + 32 * h, ov);
          } else {
            tmem_st16_sync(tmem + lane_off + kColQ + 16 * h, qv);
            tmem_st16_sync(tmem + lane_off + kColO + 16 * h, ov);
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.q_ready);
        }
        const size_t si = static_cast<size_t>(it.head) * p.total_tokens + q;
        const bool stat_in = row_in && in_bounds(si, static_cast<long long>(p.heads) * p.total_tokens);
        const float nl = stat_in ? -__ldg(p.lse + si) * kLog2e : 0.0f;
        const float drow = stat_in ? __ldg(p.delta + si) : 0.0f;
        const uint64_t nl2 = f32x2(nl, nl), d2 = f32x2(drow, drow);
        for (int j = 0; j < it.n_kv; ++j) {
          if (!warp_wait_bar(&ctl.s_full, ns & 1, abort_flag)) { ok = false; break; }
          ++ns;
          tc_fence_after_sync();
          uint32_t sr[64];
          tmem_ld64_sync(tmem + lane_off + kColS + 64 * h, sr);
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.s_free);
          const int valid = it.seg_len - j * kBlockN - 64 * h;  // keys of this half in the sample
          if (valid < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
          }
          uint64_t pp[32];
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            const uint64_t x = fma_f32x2(f32x2(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1])),
                                         sl2x2, nl2);
            float x0, x1;
            f32x2_split(x, x0, x1);
            pp[c2] = f32x2(ex2_approx(x0), ex2_approx(x1));
          }
          if (!warp_wait_bar(&ctl.dp_full, nd & 1, abort_flag)) { ok = false; break; }
          ++nd;
          tc_fence_after_sync();
          {
            uint32_t pk[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t dr[32];
              tmem_ld32_sync(tmem + lane_off + kColDP + 64 * h + 32 * half, dr);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c2 = 16 * half + i;
                const uint64_t ds = mul_f32x2(
                    pp[c2], sub_f32x2(f32x2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])), d2));
                float a, bb;
                f32x2_split(ds, a, bb);
                pk[c2] = pack_bf16x2(a, bb);
              }
            }
            tmem_st32_sync(tmem + lane_off + kColDP + 64 * h, pk);
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.ds_ready);
        }
        if (!ok) break;
        if (!warp_wait_bar(&ctl.acc_ready, pc & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const int tok0 = r0 + g4 * 32;  // token of this warp's first query row
        const int valid_rows = seg_end - tok0;
        const uint32_t stage = smem_addr(sStage) + warp * 2048;
        // bytes of one fp32 [T, H, D] tensor (the bf16 dv is half of it)
        const size_t rows_bytes = static_cast<size_t>(p.total_tokens) * p.heads * D * 4;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          const int col = h * (D / 2) + 32 * c;
          const size_t orow0 = (static_cast<size_t>(tok0) * p.heads + it.head) * D + col;
          uint32_t r[32];
          tmem_ld32_sync(tmem + lane_off + kColDQ + col, r);
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int e = 16 * k2 + 4 * v4;
              stage_put(stage, lane, v4,
                        make_uint4(__float_as_uint(__uint_as_float(r[e + 0]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 1]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 2]) * p.scale),
                                   __float_as_uint(__uint_as_float(r[e + 3]) * p.scale)));
            }
            stage_flush(stage, lane, reinterpret_cast<uint8_t*>(p.dhat + orow0 + 16 * k2),
                        static_cast<size_t>(p.heads) * D * 4, valid_rows, p.dhat, rows_bytes);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.acc_empty);
      }
    }
  }
  bwd_teardown(tmem, warp);
}

}  // namespace mf
