// Stage 2: block-diagonal (per-sample) softmax attention on the 5th-generation
// tensor cores.
//
// [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": joint
//  self-attention over packed variable-length samples with per-sample
//  cumulative offsets. The pages run it with FlashAttention's var-len
//  kernels; this kernel is its own design for sm_100a.]
//
// Persistent: one CTA per SM walks the work list with a stride of
// gridDim.x (a list laid out by mf_schedule_work gives each CTA its share of
// a longest-processing-time-first balance; its padding entries are skipped).
// A work item is 256 query rows of one head of one
// sample, split into two 128-row sub-tiles a and b that share every K/V tile
// (b is skipped when it starts past the sample end). Keys are visited in
// steps of 128.
//
//   warps 0-3 / 4-7  softmax for sub-tile a / b, one thread per query row:
//                    load the S row from TMEM, mask keys past the sample
//                    end, online max and sum in the exp2 domain, write P
//                    (bf16) back into TMEM over S, and rescale O in TMEM only
//                    when the running max of a row inside the sample grew by
//                    more than 2^8 (a stale max keeps p <= 256: exact enough
//                    in bf16, safe in fp32). At the end of an item a thread
//                    stores its row's log-normaliser (when asked), hands 1/l
//                    to the epilogue warps and goes straight on to the next
//                    item's first S.
//   warps 8-11       epilogue, one warp per TMEM lane quarter (32 rows of
//                    each sub-tile): after an item's last PV_t, O_t / l ->
//                    bf16 rows through 4 KB of shared memory per warp, so
//                    that the stores write whole 128-byte row segments
//                    (rows past the sample end are not stored); then O_t is
//                    free for the next item's first PV_t.
//   warp 12 (1 lane) TMA producer: both Q sub-tiles per item, then K_j, V_j
//                    into a ring of shared-memory stages (128-byte swizzled
//                    boxes of 128 rows x 64 dims).
//   warp 13 (1 lane) MMA issuer (also owns the TMEM allocation), one stream
//                    across item boundaries:
//                      S_a(0) S_b(0) | PV_a(j) S_a(j+1) PV_b(j) S_b(j+1) | ...
//                    where after an item's last step "j+1" is the next item's
//                    step 0, so its first S and softmax overlap the epilogue.
//                    S = Q K^T with both operands in shared memory; O += P V
//                    with P from TMEM and V (an MN-major operand) from shared
//                    memory; fp32 accumulators in TMEM. While softmax a works
//                    on S_a(j+1) the tensor core runs PV_b(j) and S_b(j+1),
//                    and the other way round.
//   warps 14-15      idle; with warps 12-13 they form warpgroup 3, which
//                    (like the epilogue warpgroup) gives registers to the
//                    softmax warpgroups (setmaxnreg: softmax 184 per thread,
//                    epilogue 64, producer and MMA 80).
//
// TMEM (512 columns): S_a [0,128) O_a [128,256) S_b [256,384) O_b [384,512).
// P_t(j) overwrites the first 64 columns of S_t after the softmax has read
// S_t(j); S_t(j+1) is issued after PV_t(j), and tcgen05 MMAs of one thread
// execute in issue order, so P is read before it is overwritten.
//
// Synchronisation (mbarriers; every arrival is waited for exactly once, in
// order, so a parity wait can never confuse two phases):
//   q_full / q_empty   producer <-> MMA, one phase per item
//   kv_full / kv_empty producer <-> MMA, per ring stage
//   s_full[t]          MMA -> softmax t, one phase per S_t. A commit tracks
//                      all earlier MMAs of the thread, so when S_t(j) lands,
//                      PV_t(j-1) is complete too: O_t may be rescaled and
//                      P_t may be overwritten without another wait.
//   p_half[t][h]       softmax t (4 warps) -> MMA, one phase per half (64
//                      keys) of P_t: the first half of PV_t starts while the
//                      softmax computes the second half's exponentials
//   o_ready[t]         MMA -> epilogue after an item's last PV_t
//   stat_ready[t]      softmax t (128 threads) -> epilogue: 1/l of each row
//   o_free[t]          epilogue (4 warps) -> MMA: O_t drained; the next
//                      item's first PV_t (which overwrites O_t) may go
//
// Every wait is bounded (kWaitLimitNs). A wait that runs out records
// MF_ERR_TIMEOUT in the device error word and raises the CTA's abort flag;
// every role leaves its loop, the producer waits (bounded) for its copies
// in flight, the MMA warp commits and waits for its MMAs, and TMEM is
// released before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/mf_attn.h"
#include "bounds.cuh"
#include "sm100_ptx.cuh"

namespace mf {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 100 ms for in-flight work on abort
constexpr int kAttnThreads = 512;
constexpr uint32_t kSoftmaxRegs = 184;   // per thread, warpgroups 0 and 1
constexpr uint32_t kEpilogueRegs = 64;   // per thread, warpgroup 2
constexpr uint32_t kControlRegs = 80;    // per thread, warpgroup 3
// The split must fit in what the CTA is launched with (512 x regs/thread):
// the host refuses to launch if the compiled kernel uses fewer registers.
constexpr int kMinLaunchRegs =
    (2 * 128 * kSoftmaxRegs + 128 * kEpilogueRegs + 128 * kControlRegs + kAttnThreads - 1) /
    kAttnThreads;
static_assert(2 * kSoftmaxRegs + kEpilogueRegs + kControlRegs <= 4 * 128,
              "the warpgroups' registers must fit the 64K register file");
constexpr int kEpilogueWarp0 = 8;  // warps 8-11
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kSubM = 128;             // rows of one query sub-tile (MMA M)
constexpr int kBlockN = MF_TILE_N;     // keys per step (MMA N of S, K of PV)
constexpr int kBoxBytes = 128 * 128;   // 128 rows x 64 bf16 = one 128-byte swizzle span
constexpr int kMaxStages = 6;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(MF_TILE_M == 2 * kSubM, "a work item is two query sub-tiles");

__device__ __forceinline__ uint32_t col_s(int t) { return 256u * static_cast<uint32_t>(t); }
__device__ __forceinline__ uint32_t col_o(int t) { return 256u * static_cast<uint32_t>(t) + 128u; }

template <int D>
struct AttnConfig {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kSubM * D * 2;  // one 128-row tile of Q, K or V
  // Deep enough that each K/V load is requested a full key step before use.
  static constexpr int kStages = D == 128 ? 4 : 6;
  // Per epilogue warp: 32 output rows x 64 dims (bf16) staged for coalesced
  // stores at the end of an item.
  static constexpr int kStageBytes = 4 * 32 * 128;
  static constexpr int kSmemBytes = kTileBytes * (2 + kStages) + kStageBytes + 1024;
  static_assert(kStages <= kMaxStages, "ring too deep");
  static_assert(kSmemBytes <= 226 * 1024, "over the 227 KB of shared memory a CTA may use");
};

struct AttnParams {
  const mf_segment* segs;
  const mf_work_item* work;
  int n_segs;
  __nv_bfloat16* out;
  float* lse;        // optional [heads, total_tokens]: natural-log softmax normaliser per row
  int n_work;
  int heads;
  int total_tokens;
  float scale_log2;  // softmax scale * log2(e)
};

struct ItemInfo {
  int seg_start;
  int seg_len;
  int head;
  int q0;      // first query row of sub-tile a
  int n_kv;    // key steps
  bool b_valid;
};

// (A work item naming a segment outside [0, n_segs) is a caller error: the
// checked build records it and uses segment 0 instead, so that every role of
// the kernel still walks the same items.)
__device__ __forceinline__ ItemInfo load_item(const mf_segment* segs, int n_segs,
                                              const mf_work_item* work, int idx) {
  const mf_work_item wi = work[idx];
  const mf_segment sg = segs[in_bounds(wi.seg, n_segs) ? wi.seg : 0];
  ItemInfo it;
  it.seg_start = sg.start;
  it.seg_len = sg.len;
  it.head = wi.head;
  it.q0 = sg.start + wi.q_tile * MF_TILE_M;
  it.n_kv = (sg.len + kBlockN - 1) / kBlockN;
  it.b_valid = it.q0 + kSubM < sg.start + sg.len;
  return it;
}

__device__ __forceinline__ ItemInfo load_item(const AttnParams& p, int idx) {
  return load_item(p.segs, p.n_segs, p.work, idx);
}

// The first work-list position >= idx in this CTA's stride that holds an
// item: a scheduled list (mf_schedule_work) pads CTAs that have fewer items
// with entries of q_tile < 0, which every role skips.
__device__ __forceinline__ int next_item(const mf_work_item* work, int n_work, int idx, int stride) {
  while (idx < n_work && work[idx].q_tile < 0) idx += stride;
  return idx;
}

struct SharedCtl {
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t kv_full[kMaxStages];
  uint64_t kv_empty[kMaxStages];
  uint64_t s_full[2];
  uint64_t p_half[2][2];  // first / second 64 keys of P_t
  uint64_t o_ready[2];
  uint64_t stat_ready[2];
  uint64_t o_free[2];
  uint64_t drain;
  float inv_l[2][kSubM];  // 1 / l of each row of the item that just ended, per sub-tile
  uint32_t tmem_base;
  int32_t abort;
};

// Inlined: a call inside a setmaxnreg region would have to fit the caller's
// register budget at every call site, which ptxas cannot arrange.
__device__ __forceinline__ bool wait_slow(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag,
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
        record_error(MF_ERR_TIMEOUT);
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

// Shared-memory descriptors are built once; a descriptor for base + off is
// the base descriptor plus off >> 4 (the start-address field is the low 14
// bits, and shared addresses stay below 256 KB, so the add never carries out
// of it). Building them per MMA would cost a dependent integer chain of ~100
// cycles on the issuing thread, longer than the 64-cycle MMA itself.

// S (tmem) = Q (smem) K^T (smem): M=128, N=128, K=D in steps of 16. Both are
// K-major with the 128-byte swizzle: a K step of 16 elements is 32 bytes
// inside a 128-byte row; 64-element column blocks are one box apart.
// (Descriptors by their low 32 bits, see mma_ss_lo.)
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(kSubM, kBlockN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = static_cast<uint32_t>(((kk / 4) * kBoxBytes + (kk % 4) * 32) >> 4);
    mma_ss_lo(d_tmem, q_lo + off, k_lo + off, kIdesc, kk > 0 ? 1u : 0u);
  }
}

// O (tmem) (+)= P (tmem, bf16) V (smem) over keys [16*k0, 16*k1): M=128, N=D,
// K=16 per MMA. V is [keys, d] with d contiguous, an MN-major operand: 16
// keys are two 8-row swizzle atoms (2 KB); 64-dim blocks are one box apart
// (the descriptor's leading byte offset).
template <int D, int k0, int k1>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo,
                                         bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(kSubM, D, 0, 1);
#pragma unroll
  for (int kk = k0; kk < k1; ++kk)
    mma_ts_lo(o_tmem, p_tmem + kk * 8, v_lo + static_cast<uint32_t>(kk * (2048 >> 4)), kIdesc,
              (accumulate || kk > 0) ? 1u : 0u);
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
  uint8_t* sQ = smem;                // sub-tile a, then sub-tile b
  uint8_t* sKV = smem + 2 * kTile;   // NS stages
  uint8_t* sOut = sKV + NS * kTile;  // output staging, 4 KB per epilogue warp
  volatile int32_t* abort_flag = &ctl.abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.s_full[t], 1);
      mbar_init(&ctl.p_half[t][0], 4);
      mbar_init(&ctl.p_half[t][1], 4);
      mbar_init(&ctl.o_ready[t], 1);
      mbar_init(&ctl.stat_ready[t], kSubM);
      mbar_init(&ctl.o_free[t], 4);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;
  const int stride = static_cast<int>(gridDim.x);
  // Each warpgroup re-splits its registers first thing in its own branch, so
  // that the code of every role is compiled under its own budget:
  // warpgroup 3 (producer, MMA issuer, two idle warps) and warpgroup 2
  // (epilogue) give registers to warpgroups 0 and 1 (softmax).
  if (warp >= 12) {
    setmaxnreg_dec<kControlRegs>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------ TMA producer ---
    if (lane == 0) {
      int g = 0;  // tile loads issued into the ring so far
      int k = 0;  // items started
      bool ok = true;
      for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
           idx = next_item(p.work, p.n_work, idx + stride, stride), ++k) {
        const ItemInfo it = load_item(p, idx);
        // Tiles start inside the tensor (a tile may run past its end: TMA
        // fills the rows past T with zeros).
        if (kChecked) {
          in_bounds(it.head, p.heads);
          in_bounds(it.q0, p.total_tokens);
          in_bounds(it.seg_start + it.seg_len - 1, p.total_tokens);
        }
        if (k > 0 && !wait_bar(&ctl.q_empty, (k - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&ctl.q_full, 2 * kTile);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int b = 0; b < Cfg::kBoxes; ++b)
            tma_load_3d(sQ + t * kTile + b * kBoxBytes, &tmap_q, &ctl.q_full, 64 * b, it.head,
                        it.q0 + t * kSubM);
        for (int j = 0; j < it.n_kv && ok; ++j) {
          for (int which = 0; which < 2; ++which, ++g) {
            const int st = g % NS;
            if (!wait_bar(&ctl.kv_empty[st], ((g / NS) & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&ctl.kv_full[st], kTile);
            const CUtensorMap* map = which ? &tmap_v : &tmap_k;
#pragma unroll
            for (int b = 0; b < Cfg::kBoxes; ++b)
              tma_load_3d(sKV + st * kTile + b * kBoxBytes, map, &ctl.kv_full[st], 64 * b, it.head,
                          it.seg_start + j * kBlockN);
          }
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        if (k > 0) wait_slow(&ctl.q_full, (k - 1) & 1, nullptr, kDrainLimitNs);
        for (int i = g - NS > 0 ? g - NS : 0; i < g; ++i)
          wait_slow(&ctl.kv_full[i % NS], (i / NS) & 1, nullptr, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------- MMA issuer ---
    if (lane == 0) {
      const uint32_t q_desc[2] = {smem_desc_sw128_lo(smem_addr(sQ), 16),
                                  smem_desc_sw128_lo(smem_addr(sQ + kTile), 16)};
      // K stages as K-major operands, V stages as MN-major operands.
      const uint32_t k_desc0 = smem_desc_sw128_lo(smem_addr(sKV), 16);
      const uint32_t v_desc0 = smem_desc_sw128_lo(smem_addr(sKV), kBoxBytes);
      constexpr uint32_t kStageStep = static_cast<uint32_t>(kTile >> 4);
      // Loads this CTA will consume: a stage is released only if it will be
      // refilled, so that no arrival is left pending when the CTA exits.
      int total_loads = 0;
      for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work;
           idx = next_item(p.work, p.n_work, idx + stride, stride))
        total_loads += 2 * load_item(p, idx).n_kv;
      int g = 0;                 // tile loads consumed so far
      int k = 0;                 // current item's index among this CTA's items
      uint32_t np[2] = {0, 0};   // P phases consumed per sub-tile
      uint32_t nused[2] = {0, 0};  // items whose O_t went to the epilogue
      bool ok = true;
      int idx = next_item(p.work, p.n_work, blockIdx.x, stride);
      if (idx < p.n_work) {
        ItemInfo it = load_item(p, idx);
        int nidx = next_item(p.work, p.n_work, idx + stride, stride);
        // S_t(0) of the first item.
        {
          const int st = g % NS;
          ok = wait_bar(&ctl.q_full, 0, abort_flag) &&
               wait_bar(&ctl.kv_full[st], (g / NS) & 1, abort_flag);
          if (ok) {
            tc_fence_after_sync();
            for (int t = 0; t < (it.b_valid ? 2 : 1); ++t) {
              issue_qk<D>(tmem + col_s(t), q_desc[t], k_desc0 + st * kStageStep);
              mma_commit(&ctl.s_full[t]);
            }
            if (it.n_kv == 1 && nidx < p.n_work) mma_commit(&ctl.q_empty);
            if (g + NS < total_loads) mma_commit(&ctl.kv_empty[st]);
            ++g;
          }
        }
        // One stream of steps across items: step j issues PV_t(j) and the
        // S_t of the following step, which after an item's last step is the
        // next item's step 0.
        while (ok) {
          const bool has_next = nidx < p.n_work;
          const ItemInfo nx = has_next ? load_item(p, nidx) : it;
          for (int j = 0; j < it.n_kv && ok; ++j) {
            const bool last = j + 1 == it.n_kv;
            const bool s_next = !last || has_next;  // an S follows this step
            // the item that S belongs to: its sub-tile b, its last step
            const bool s_b = last ? nx.b_valid : it.b_valid;
            const bool s_is_last = last ? nx.n_kv == 1 : j + 2 == it.n_kv;
            const int gv = g;      // V_j
            const int gk = g + 1;  // the following K
            const int sv = gv % NS, sk = gk % NS;
            if (!wait_bar(&ctl.kv_full[sv], (gv / NS) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
            bool k_ready = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (t == 0 || it.b_valid) {
                if (j == 0 && nused[t] > 0) {
                  // O_t still holds the previous item's output: the first
                  // PV_t overwrites it only once the epilogue has drained it.
                  if (!wait_bar(&ctl.o_free[t], (nused[t] - 1) & 1, abort_flag)) { ok = false; break; }
                }
                // PV in two halves: the first 64 keys start while the softmax
                // is still computing the exponentials of the second 64.
                if (!wait_bar(&ctl.p_half[t][0], np[t] & 1, abort_flag)) { ok = false; break; }
                tc_fence_after_sync();
                issue_pv<D, 0, 4>(tmem + col_o(t), tmem + col_s(t), v_desc0 + sv * kStageStep, j > 0);
                if (!wait_bar(&ctl.p_half[t][1], np[t] & 1, abort_flag)) { ok = false; break; }
                ++np[t];
                tc_fence_after_sync();
                issue_pv<D, 4, 8>(tmem + col_o(t), tmem + col_s(t), v_desc0 + sv * kStageStep, true);
                if (last) {
                  mma_commit(&ctl.o_ready[t]);
                  ++nused[t];
                }
              }
              if (s_next && (t == 0 || s_b)) {
                if (!k_ready) {
                  // The following K is needed only now, after PV_a(j) has
                  // been queued; a new item's first S also needs its Q.
                  if (!wait_bar(&ctl.kv_full[sk], (gk / NS) & 1, abort_flag)) { ok = false; break; }
                  if (last && !wait_bar(&ctl.q_full, (k + 1) & 1, abort_flag)) { ok = false; break; }
                  tc_fence_after_sync();
                  k_ready = true;
                }
                issue_qk<D>(tmem + col_s(t), q_desc[t], k_desc0 + sk * kStageStep);
                mma_commit(&ctl.s_full[t]);
              }
            }
            if (!ok) break;
            if (gv + NS < total_loads) mma_commit(&ctl.kv_empty[sv]);
            g = gv + 1;
            if (s_next) {
              // Q is free once the last S of its item has been issued (the
              // producer then loads the next item's Q over it).
              const bool after = last ? (nidx < p.n_work &&
                                         next_item(p.work, p.n_work, nidx + stride, stride) < p.n_work)
                                      : has_next;
              if (s_is_last && after) mma_commit(&ctl.q_empty);
              if (gk + NS < total_loads) mma_commit(&ctl.kv_empty[sk]);
              g = gk + 1;
            }
          }
          if (!ok || !has_next) break;
          it = nx;
          idx = nidx;
          nidx = next_item(p.work, p.n_work, idx + stride, stride);
          ++k;
        }
      }
      if (!ok) {
        // Every MMA issued so far must finish before TMEM is released.
        mma_commit(&ctl.drain);
        wait_slow(&ctl.drain, 0, nullptr, kDrainLimitNs);
      }
    }
  }
  } else if (warp < 8) {
    // ----------------------------------------------------------- softmax ---
    setmaxnreg_inc<kSoftmaxRegs>();
    const int t = warp / 4;  // sub-tile
    const int wl = warp % 4;
    const int row = wl * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const uint32_t s_tmem = tmem + lane_off + col_s(t);
    const uint32_t o_tmem = tmem + lane_off + col_o(t);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    uint32_t ns = 0;  // S phases consumed
    bool ok = true;
    for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
         idx = next_item(p.work, p.n_work, idx + stride, stride)) {
      const ItemInfo it = load_item(p, idx);
      if (t == 1 && !it.b_valid) continue;
      // Rows past the sample end (another sample's tokens, or zeros) are
      // computed but never stored, and they take no part in the rescale vote:
      // a sample's output then depends on its own tokens only, whatever it is
      // packed with.
      const bool row_in = it.q0 + t * kSubM + row < it.seg_start + it.seg_len;
      float m = -INFINITY;  // running max of s * scale * log2(e)
      float l = 0.0f;       // running sum of p
      for (int j = 0; j < it.n_kv; ++j) {
        if (!warp_wait_bar(&ctl.s_full[t], ns & 1, abort_flag)) { ok = false; break; }
        ++ns;
        tc_fence_after_sync();
        float s[128];
        {
          uint32_t sr[128];
          tmem_ld64x2_sync(s_tmem, sr);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
        }
        const int valid = it.seg_len - j * kBlockN;  // keys of this step inside the sample
        if (valid < kBlockN) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
        float mx2 = fmax3(s[6], s[7], s[8]), mx3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
        for (int c = 12; c < 124; c += 8) {
          mx0 = fmax3(mx0, s[c], s[c + 1]);
          mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
          mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
          mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
        }
        mx0 = fmax3(mx0, s[124], s[125]);
        mx1 = fmax3(mx1, s[126], s[127]);
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
        const float m_new = fmaxf(m, m_tile);
        if (j == 0 || __any_sync(0xffffffffu, row_in && m_new > m + kRescaleThreshold)) {
          // S_t(j) has landed, so PV_t(j-1) is complete: O_t may be rescaled.
          const float factor = ex2_approx(m - m_new);  // 0 on the first step
          l *= factor;
          if (j > 0) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32_sync(o_tmem + 32 * c, r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
              tmem_st32_sync(o_tmem + 32 * c, r);
            }
          }
          m = m_new;
        }
        const uint64_t neg_m = f32x2(-m, -m);
        float la0 = 0.f, la1 = 0.f, lb0 = 0.f, lb1 = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int e = 64 * h + 2 * c;
            const uint64_t x = fma_f32x2(f32x2(s[e], s[e + 1]), sl2x2, neg_m);
            float x0, x1;
            f32x2_split(x, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            // Row sum in four scalar chains (packing p0, p1 for a paired add
            // would cost register moves).
            if (c & 1) { la1 += p0; lb1 += p1; } else { la0 += p0; lb0 += p1; }
            pk[c] = pack_bf16x2(p0, p1);
          }
          // P over the first 64 columns of S, 32 columns (64 keys) at a time.
          tmem_st32_sync(s_tmem + 32 * h, pk);
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.p_half[t][h]);
        }
        l += (la0 + la1) + (lb0 + lb1);
      }
      if (!ok) break;
      // ---- end of the item: the row's log-normaliser, and 1/l for the
      // epilogue warps, which drain O_t while this warp starts the next item.
      const int q_row = it.q0 + t * kSubM + row;
      // log of the row's softmax normaliser, sum_u exp(s_u * scale), for the
      // backward pass: m and l are in the exp2 domain of s * scale * log2(e).
      if (p.lse && row_in) {
        const size_t li = static_cast<size_t>(it.head) * p.total_tokens + q_row;
        if (in_bounds(li, static_cast<long long>(p.heads) * p.total_tokens))
          p.lse[li] = (m + log2f(l)) * 0.6931471805599453f;
      }
      ctl.inv_l[t][row] = 1.0f / l;
      mbar_arrive(&ctl.stat_ready[t]);
    }
  } else {
    // ---------------------------------------------------------- epilogue ---
    setmaxnreg_dec<kEpilogueRegs>();
    const int wq = warp % 4;  // TMEM lane quarter: rows 32 * wq .. of each sub-tile
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* stage = sOut + (warp - kEpilogueWarp0) * 4096;
    const int rr0 = lane >> 3;  // first row this lane stores, then every 4th
    const int cc = lane & 7;    // 16-byte chunk of the row this lane stores
    uint32_t no[2] = {0, 0};    // items drained per sub-tile
    bool ok = true;
    for (int idx = next_item(p.work, p.n_work, blockIdx.x, stride); idx < p.n_work && ok;
         idx = next_item(p.work, p.n_work, idx + stride, stride)) {
      const ItemInfo it = load_item(p, idx);
      const int row_end = it.seg_start + it.seg_len;
      for (int t = 0; t < (it.b_valid ? 2 : 1); ++t) {
        if (!warp_wait_bar(&ctl.stat_ready[t], no[t] & 1, abort_flag) ||
            !warp_wait_bar(&ctl.o_ready[t], no[t] & 1, abort_flag)) {
          ok = false;
          break;
        }
        ++no[t];
        tc_fence_after_sync();
        const float inv_l = ctl.inv_l[t][row];
        const uint32_t o_tmem = tmem + lane_off + col_o(t);
        const int row0 = it.q0 + t * kSubM + wq * 32;  // token of the warp's first row
        // O / l in 64-dim halves through this warp's 4 KB of shared memory:
        // each lane writes its row (128 bytes, 16-byte chunk c at c ^ (row % 8)),
        // then each store instruction of the warp writes four whole 128-byte
        // row segments (eight lanes per row) instead of 32 scattered 16-byte
        // pieces.
#pragma unroll 1
        for (int half = 0; half < D / 64; ++half) {
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            uint32_t r[16];
            tmem_ld16_sync(o_tmem + 64 * half + 16 * c16, r);
#pragma unroll
            for (int v4 = 0; v4 < 2; ++v4) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v4 + 0]) * inv_l, __uint_as_float(r[8 * v4 + 1]) * inv_l);
              o.y = pack_bf16x2(__uint_as_float(r[8 * v4 + 2]) * inv_l, __uint_as_float(r[8 * v4 + 3]) * inv_l);
              o.z = pack_bf16x2(__uint_as_float(r[8 * v4 + 4]) * inv_l, __uint_as_float(r[8 * v4 + 5]) * inv_l);
              o.w = pack_bf16x2(__uint_as_float(r[8 * v4 + 6]) * inv_l, __uint_as_float(r[8 * v4 + 7]) * inv_l);
              const int c = 2 * c16 + v4;
              *reinterpret_cast<uint4*>(stage + lane * 128 + ((c ^ (lane & 7)) << 4)) = o;
            }
          }
          if (half == D / 64 - 1) {
            // O_t has been read: the next item's first PV_t may overwrite it.
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.o_free[t]);
          }
          __syncwarp();
#pragma unroll 2
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + rr0;
            const uint4 o = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((cc ^ (rr & 7)) << 4));
            const int tok = row0 + rr;
            const size_t oi = (static_cast<size_t>(tok) * p.heads + it.head) * (D / 8) + 8 * half + cc;
            if (tok < row_end &&
                in_bounds(oi, static_cast<long long>(p.total_tokens) * p.heads * (D / 8)))
              reinterpret_cast<uint4*>(p.out)[oi] = o;
          }
          __syncwarp();
        }
      }
    }
  }

  // ---------------------------------------------------------- teardown ---
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mf
