/*
 * mf_attn.h -- C ABI of the packed joint text+image attention forward
 * (the attention hot path of Mage-Flow's Native-Resolution MMDiT), for
 * NVIDIA B200 (sm_100a).
 *
 * The operation. Images of different resolutions and aspect ratios are
 * flattened to latent token sequences and packed, with their variable-length
 * text tokens, into one buffer without padding; attention runs inside each
 * sample only, which per-sample cumulative offsets (cu_seqlens) describe
 * [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)";
 * video overview, 00:03:16-00:04:03]. Text and image streams are normalised
 * with separate parameters before the joint self-attention [same section:
 * modality-specific normalization], and image tokens carry per-sample 2D
 * rotary position embeddings [video overview, 00:03:16; capabilities page,
 * "Key Capabilities"].
 *
 * Readings this library adopts where the pages give no formula:
 *  - Sample layout: n_text text tokens, then `frames` latent grids of
 *    grid_h x grid_w tokens, each flattened row-major. An editing sample has
 *    frames = 2 (target, then reference); every frame uses the same grid
 *    positions.
 *  - Normalisation: RMSNorm over head_dim for each (token, head) of q and k,
 *    x * rsqrt(mean(x^2) + eps) * gamma, with four gamma vectors of length
 *    head_dim (q/k x text/image) shared by all heads. V is untouched.
 *  - 2D RoPE, after the norm, image tokens only: grid row r rotates dims
 *    [0, d/2), grid column c rotates dims [d/2, d), in adjacent pairs
 *    (2j, 2j+1) by pos * 10000^(-2j/(d/2)). Text tokens are not rotated.
 *    The *_3d entry points add a frame axis (see there).
 *  - Attention: non-causal softmax(q_hat k_hat^T * scale) v within a sample.
 *
 * Conventions for every entry point:
 *  - Errors are returned as mf_status; nothing aborts, throws or prints.
 *  - Device entry points are asynchronous on the caller's stream (`stream` is
 *    a cudaStream_t; NULL is the legacy default stream) and allocate nothing,
 *    so they can be captured in a CUDA graph.
 *  - All device pointers are owned by the caller; inputs are never written.
 *  - Launch failures return MF_ERR_CUDA. A fault the kernels detect while
 *    running (a pipeline wait that exceeded its time limit) is recorded on
 *    the device and reported by mf_get_device_error().
 *  - libmfattn_checked.so, built from the same sources with -DMF_CHECKED,
 *    exports the same calls. Its prologue, attention and backward kernels
 *    compare every global index they compute with the extent of its buffer
 *    before the access; an index outside records MF_ERR_BOUNDS (reported by
 *    mf_get_device_error) and the access is skipped. The sub-layer's GEMM,
 *    adaLN and table kernels are not checked. The product library,
 *    libmfattn.so, compiles the checks away.
 */
#ifndef MF_ATTN_H
#define MF_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MF_OK = 0,
  MF_ERR_INVALID_ARG = -1, /* NULL pointer, negative or inconsistent size      */
  MF_ERR_UNSUPPORTED = -2, /* head_dim not in {64, 128}                         */
  MF_ERR_ALIGNMENT = -3,   /* a device pointer is not 16-byte aligned           */
  MF_ERR_WORKSPACE = -4,   /* workspace smaller than the *_workspace_bytes query  */
  MF_ERR_BUDGET = -5,      /* total tokens exceed the pack's token budget       */
  MF_ERR_CUDA = -6,        /* a CUDA runtime or driver call failed              */
  MF_ERR_TIMEOUT = -7,     /* a kernel pipeline wait ran out of time            */
  MF_ERR_BOUNDS = -8       /* checked build only: a kernel computed a global
                              index outside its buffer (the access was skipped) */
} mf_status;

/* One packed sample: tokens [start, start + len) of the pack. 24 bytes. */
typedef struct {
  int32_t start;
  int32_t len;    /* n_text + frames * grid_h * grid_w */
  int32_t n_text;
  int32_t grid_h; /* latent rows    */
  int32_t grid_w; /* latent columns */
  int32_t frames;
} mf_segment;

/* One unit of attention work: query rows
 * [segs[seg].start + q_tile * MF_TILE_M, min(+MF_TILE_M, segment end)) of head `head`,
 * attending over all kv_len keys of the sample. 16 bytes. The kernel splits
 * an item into two 128-row tensor-core tiles that share every K/V tile. */
typedef struct {
  int32_t seg;
  int32_t head;
  int32_t q_tile;
  int32_t kv_len;
} mf_work_item;

#define MF_TILE_M 256 /* query rows per work item */
#define MF_TILE_N 128 /* keys per pipeline step   */

/* ABI version of this header (incremented on any change of signature). */
int32_t mf_abi_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char* mf_status_string(mf_status status);

/*
 * mf_pack_plan -- host only; builds the per-sample layout and the work list.
 * [Mage-Flow summary, "Native-Resolution MMDiT": packing under a fixed token
 *  budget with per-sample cumulative offsets; video overview, 00:04:03: zero
 *  padding.]
 *
 * Inputs (host arrays of n_samples entries each):
 *   n_text[i] >= 0, grid_h[i] >= 1, grid_w[i] >= 1, frames[i] >= 1
 *   (frames == NULL means 1 for every sample). heads >= 1.
 *   head_dim must be 64 or 128 (checked here so a plan never describes work
 *   the kernels cannot run). token_budget <= 0 means no budget.
 * Outputs (host, caller-owned; each may be NULL to skip it):
 *   cu_seqlens [n_samples + 1]   prefix sums of the sample lengths, int32
 *   segs       [n_samples]       mf_segment per sample
 *   work       [*n_work]         work items ordered by cost, largest first:
 *                                sample length x 128-row query sub-tiles in
 *                                the item (ties: sample index, head, q_tile)
 *   n_work, total_tokens         scalars (may be NULL)
 * Two-call convention: call with work == NULL to learn *n_work, then again
 * with *n_work set to the capacity of `work` (at least the count returned);
 * *n_work then receives the count written. A non-NULL `work` needs a non-NULL
 * n_work. The sum of the lengths is exact: no rounding of segments to tiles,
 * no padding tokens.
 * Errors: MF_ERR_INVALID_ARG for a bad count, size or NULL input array, or a
 * total that does not fit int32; MF_ERR_UNSUPPORTED for head_dim;
 * MF_ERR_BUDGET when the total exceeds token_budget (> 0).
 */
mf_status mf_pack_plan(int32_t n_samples, const int32_t* n_text, const int32_t* grid_h,
                       const int32_t* grid_w, const int32_t* frames, int32_t heads,
                       int32_t head_dim, int64_t token_budget, int32_t* cu_seqlens,
                       mf_segment* segs, mf_work_item* work, int32_t* n_work,
                       int32_t* total_tokens);

/*
 * mf_schedule_work -- host only; assigns a work list to n_ctas persistent
 * CTAs ahead of time, longest processing time first: items in decreasing
 * cost (key steps x 20 with two query sub-tiles, x 19 with one: a lone
 * sub-tile's step is the softmax -> PV -> next-S chain by itself, about 95 %
 * of a two-sub-tile step; ties keep the input order), each to the CTA with
 * the least work so far (lowest index on ties). The result is laid out
 * for the kernels' traversal, in which CTA c takes positions c, c + n_ctas,
 * c + 2 n_ctas, ...: position r * n_ctas + c holds CTA c's r-th item, and a
 * CTA with fewer items than the busiest is padded with {0, 0, -1, 0}
 * entries (q_tile < 0), which every kernel skips. Launched on any other
 * number of CTAs the list stays correct (every item runs once), only the
 * balance is lost; the library launches min(n_work, SM count) CTAs.
 *   work, n_work   a work list from mf_pack_plan (host)
 *   n_ctas         CTAs to balance over (>= 1; capped at n_work)
 *   sched          [*n_sched] output (host, caller-owned), or NULL
 *   n_sched        with sched == NULL receives the length; otherwise the
 *                  capacity of sched on entry and the length written on exit
 * Errors: MF_ERR_INVALID_ARG for NULL arguments, n_work < 1, n_ctas < 1,
 * an input entry with q_tile < 0, or too small a capacity.
 */
mf_status mf_schedule_work(const mf_work_item* work, int32_t n_work, int32_t n_ctas,
                           mf_work_item* sched, int32_t* n_sched);

/*
 * mf_joint_attn_workspace_bytes -- bytes of device workspace mf_joint_attn_fwd
 * (and its stages) needs: the normalised, rotated q_hat and k_hat
 * ([T, H, d] bf16 each, each padded to a multiple of 256 bytes).
 * Returns 0 for invalid sizes.
 */
size_t mf_joint_attn_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim);

/*
 * mf_qk_prologue -- stage 1 of mf_joint_attn_fwd, exposed for measurement.
 * For every token and head, RMSNorm q and k with the gamma of the token's
 * modality and rotate image tokens by their grid position (see the readings
 * above); writes q_hat and k_hat (bf16, [T, H, d]) into the workspace.
 *   q, k           bf16 [total_tokens, heads, head_dim], contiguous, 16-B aligned
 *   g_q_text ...   fp32 [head_dim] each, device
 *   cu_seqlens_dev int32 [n_samples + 1], device, from mf_pack_plan
 *   segs_dev       mf_segment [n_samples], device, from mf_pack_plan
 *   eps            added to the mean square (e.g. 1e-6), must be >= 0
 *   workspace      device, >= mf_joint_attn_workspace_bytes(...), 256-B aligned
 */
mf_status mf_qk_prologue(const void* q, const void* k, const float* g_q_text,
                         const float* g_q_img, const float* g_k_text, const float* g_k_img,
                         const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                         int32_t n_samples, int32_t total_tokens, int32_t heads,
                         int32_t head_dim, float eps, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * mf_packed_attention -- stage 2 of mf_joint_attn_fwd, exposed for
 * measurement: block-diagonal softmax attention of q_hat, k_hat (read from
 * the workspace that mf_qk_prologue filled) and v, on tensor cores.
 *   v              bf16 [total_tokens, heads, head_dim], contiguous, 16-B aligned
 *   work_dev       mf_work_item [n_work], device, from mf_pack_plan, or laid
 *                  out by mf_schedule_work (entries with q_tile < 0 are skipped)
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim)
 *   out            bf16 [total_tokens, heads, head_dim], 16-B aligned, must not
 *                  overlap q, k, v or the workspace
 */
mf_status mf_packed_attention(const void* v, const mf_segment* segs_dev, int32_t n_samples,
                              const mf_work_item* work_dev, int32_t n_work, int32_t total_tokens,
                              int32_t heads, int32_t head_dim, float softmax_scale, void* out,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * mf_joint_attn_fwd -- the whole forward: mf_qk_prologue then
 * mf_packed_attention on `stream`. Arguments as described above.
 */
mf_status mf_joint_attn_fwd(const void* q, const void* k, const void* v, const float* g_q_text,
                            const float* g_q_img, const float* g_k_text, const float* g_k_img,
                            const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                            int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
                            int32_t total_tokens, int32_t heads, int32_t head_dim, float eps,
                            float softmax_scale, void* out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * mf_qk_prologue_3d, mf_joint_attn_fwd_3d -- the same two calls with a 3D
 * rotary embedding: a frame axis next to the grid row and column, so that
 * the frames of an editing sample (target, then source) are told apart by
 * position [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)",
 * Conditioning: source image latents are concatenated with the target
 * latents under a 3D RoPE with a frame dimension].
 * Reading (the pages give no split of head_dim among the axes): dims
 * [0, frame_dims) rotate by the token's frame index f (the sample's grids
 * counted from 0: target 0, source 1), then two parts of
 * S = (head_dim - frame_dims) / 2 dims rotate by the grid row r and by the
 * grid column c. Each part rotates its adjacent pairs (2j, 2j+1) by
 * pos * 10000^(-2j / width), width being that part's number of dims
 * (frame_dims or S). Text tokens are not rotated. frame_dims = 0 is the 2D
 * rotation of mf_qk_prologue / mf_joint_attn_fwd, bit for bit.
 *   frame_dims  a multiple of 4 with 0 <= frame_dims <= head_dim - 4
 *               (so that every part holds whole pairs); otherwise
 *               MF_ERR_INVALID_ARG.
 * Every other argument, and the errors, as for mf_qk_prologue and
 * mf_joint_attn_fwd.
 */
mf_status mf_qk_prologue_3d(const void* q, const void* k, const float* g_q_text,
                            const float* g_q_img, const float* g_k_text, const float* g_k_img,
                            const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                            int32_t n_samples, int32_t total_tokens, int32_t heads,
                            int32_t head_dim, float eps, int32_t frame_dims, void* workspace,
                            size_t workspace_bytes, void* stream);

mf_status mf_joint_attn_fwd_3d(const void* q, const void* k, const void* v,
                               const float* g_q_text, const float* g_q_img,
                               const float* g_k_text, const float* g_k_img,
                               const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                               int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
                               int32_t total_tokens, int32_t heads, int32_t head_dim, float eps,
                               int32_t frame_dims, float softmax_scale, void* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Training: the forward with its per-row log-normaliser, and the backward.
 * [The pages measure their fused-kernel speedup on training the NR-MMDiT:
 *  video overview, 00:05:08; paper summary, "Training Infrastructure".]
 *
 * mf_joint_attn_fwd_lse -- mf_joint_attn_fwd_3d that also writes
 *   lse     fp32 [heads, total_tokens] (head-major), device, 4-B aligned:
 *           lse[h, t] = log(sum_u exp(scale * q_hat_t . k_hat_u)) over the
 *           keys u of t's sample (natural log). The backward needs it.
 *
 * mf_bwd_workspace_bytes -- device workspace mf_joint_attn_bwd needs
 *   (q_hat, k_hat, the row terms D = rowsum(dout * out), fp32 dq_hat and
 *   dk_hat, and the per-block gamma-gradient partials). 0 for invalid sizes.
 *
 * mf_joint_attn_bwd -- gradients of the forward for dL/dout = dout:
 *   inputs   q, k, v, the four gammas, the plan arrays, eps, frame_dims and
 *            softmax_scale exactly as given to the forward; out (bf16
 *            [T, H, d]) and lse as the forward wrote them; dout (bf16
 *            [T, H, d], 16-B aligned).
 *   outputs  dq, dk, dv (bf16 [T, H, d], 16-B aligned) and dgamma (fp32
 *            [4, head_dim] in the order q_text, q_img, k_text, k_img: each
 *            summed over all tokens and heads of its role and modality).
 *            Outputs must not overlap the inputs, the workspace or one
 *            another (MF_ERR_INVALID_ARG).
 *   The chain rule through the attention (dS = P * (dP - D)), the rotation
 *   (transposed) and the RMSNorm. Every result is deterministic: no atomics;
 *   the gamma sums run in a fixed order. Asynchronous on `stream`.
 *   Errors as for mf_joint_attn_fwd_3d; MF_ERR_WORKSPACE when
 *   workspace_bytes < mf_bwd_workspace_bytes(...).
 */
mf_status mf_joint_attn_fwd_lse(const void* q, const void* k, const void* v,
                                const float* g_q_text, const float* g_q_img,
                                const float* g_k_text, const float* g_k_img,
                                const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                                int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
                                int32_t total_tokens, int32_t heads, int32_t head_dim, float eps,
                                int32_t frame_dims, float softmax_scale, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

size_t mf_bwd_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim);

mf_status mf_joint_attn_bwd(const void* q, const void* k, const void* v, const float* g_q_text,
                            const float* g_q_img, const float* g_k_text, const float* g_k_img,
                            const void* out, const void* dout, const float* lse,
                            const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                            int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
                            int32_t total_tokens, int32_t heads, int32_t head_dim, float eps,
                            int32_t frame_dims, float softmax_scale, void* dq, void* dk, void* dv,
                            float* dgamma, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The joint-attention sub-layer around the path, forward: adaLN modulation,
 * per-modality QKV projection (bias, QK-RMSNorm and rotation fused into the
 * GEMM's epilogue), the packed joint attention, per-modality output
 * projection (bias, gate and residual fused into the GEMM's epilogue).
 * [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": an MMDiT
 *  with modality-specific normalization and joint self-attention; "Training
 *  Infrastructure": adaptive normalization / RoPE / gating fused into CUDA
 *  kernels.] Readings (the pages give no formula): adaLN as in DiT, text and
 * image streams with their own parameters as in an MMDiT. For token t of
 * sample s, modality m (0 text, 1 image), C = heads * head_dim:
 *   x_t  = LN(h_t) * (1 + scale[s,m]) + shift[s,m]   (LN over C, no affine, eps_ln)
 *   qkv  = W_qkv[m] x_t + b_qkv[m]; q, k, v = the three C-wide thirds, viewed
 *          [heads, head_dim]; q and k through the RMSNorm / rotation of
 *          mf_qk_prologue_3d (eps, frame_dims)
 *   o    = the packed joint attention (softmax_scale as mf_joint_attn_fwd)
 *   h'_t = h_t + gate[s,m] * (W_o[m] o_t + b_o[m])
 * Arguments (device, 16-B aligned unless noted):
 *   h, h_out            bf16 [T, C]; h_out must not overlap h or the workspace
 *   shift, scale, gate  fp32 [n_samples, 2, C]
 *   w_qkv, b_qkv        bf16 [2, 3C, C] (row n of W is output n), fp32 [2, 3C]
 *   w_o, b_o            bf16 [2, C, C], fp32 [2, C]
 *   gammas, plan arrays, eps, frame_dims, softmax_scale as mf_joint_attn_fwd_3d
 *   workspace           >= mf_block_workspace_bytes(T, heads, head_dim), 256-B aligned
 * MF_ERR_UNSUPPORTED unless head_dim is 64 or 128 and C is a multiple of 128
 * and at most 4096. Asynchronous on `stream`.
 */
size_t mf_block_workspace_bytes(int32_t total_tokens, int32_t heads, int32_t head_dim);

mf_status mf_attn_block_fwd(const void* h, const float* shift, const float* scale,
                            const float* gate, const void* w_qkv, const float* b_qkv,
                            const void* w_o, const float* b_o, const float* g_q_text,
                            const float* g_q_img, const float* g_k_text, const float* g_k_img,
                            const int32_t* cu_seqlens_dev, const mf_segment* segs_dev,
                            int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
                            int32_t total_tokens, int32_t heads, int32_t head_dim, float eps_ln,
                            float eps, int32_t frame_dims, float softmax_scale, void* h_out,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * mf_joint_attn_fwd_static_scratch -- the same forward for callers that
 * cannot allocate device memory at all. The paper has no counterpart to this
 * entry point; it exists for how the library is called, not for the method.
 *
 * Who needs it: code that is handed a stream but no allocator -- a plugin
 * inside a host framework that owns every byte of device memory, a caller in
 * the middle of a global-mode stream capture (where cudaMalloc is illegal),
 * or a latency-critical loop that cannot pay for cudaMalloc's implicit device
 * synchronisation -- and so cannot provide the workspace mf_joint_attn_fwd
 * asks for.
 *
 * Instead of a caller workspace it uses a scratch array of
 * MF_STATIC_SCRATCH_BYTES bytes that lives in the library itself (a
 * file-scope device array): every GPU that loads the library holds those
 * bytes until the process exits. This entry point allocates nothing and
 * calls no allocating routine. Arguments are those of mf_joint_attn_fwd
 * without workspace / workspace_bytes; inputs and outputs are still the
 * caller's.
 *   - Packs whose scratch need, mf_joint_attn_workspace_bytes(total_tokens,
 *     heads, head_dim), exceeds MF_STATIC_SCRATCH_BYTES are rejected with
 *     MF_ERR_WORKSPACE before anything is launched (64 MiB holds q_hat and
 *     k_hat for up to ~131,000 (token, head) rows at head_dim 128).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins. The address is kept once a lookup
 *     has succeeded (a failed lookup returns MF_ERR_CUDA and is retried by
 *     the next call). cudaDeviceReset unloads the library's device code and
 *     with it the array: after a reset of a device, do not call this entry
 *     point on that device again in the same process.
 *   - All calls share the one array, and it keeps whatever the last call
 *     left in it (every call rewrites the parts it reads). Calls whose
 *     kernels overlap on the GPU -- on two streams, or from two threads --
 *     race on the array: serialise them.
 */
#define MF_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

mf_status mf_joint_attn_fwd_static_scratch(
    const void* q, const void* k, const void* v, const float* g_q_text, const float* g_q_img,
    const float* g_k_text, const float* g_k_img, const int32_t* cu_seqlens_dev,
    const mf_segment* segs_dev, int32_t n_samples, const mf_work_item* work_dev, int32_t n_work,
    int32_t total_tokens, int32_t heads, int32_t head_dim, float eps, float softmax_scale,
    void* out, void* stream);

/*
 * mf_selftest_exp2 -- diagnostic: y[i] = 2^x[i] computed by the same
 * instruction the attention softmax uses for its exponentials (the MUFU
 * unit's approximate exp2, denormal results flushed to zero), so that its
 * accuracy can be checked on its own. x, y: device fp32 arrays of n elements
 * (n >= 0). Asynchronous on `stream`; MF_ERR_INVALID_ARG for NULL pointers
 * or n < 0.
 */
mf_status mf_selftest_exp2(const float* x, float* y, int32_t n, void* stream);

/*
 * mf_selftest_timeout -- diagnostic for the failure path: launches one CTA
 * whose thread 0 waits, through the same bounded wait the attention kernel
 * uses, on an mbarrier that nothing ever arrives on. After limit_ns
 * nanoseconds (1 <= limit_ns <= 10^9) the wait gives up, records
 * MF_ERR_TIMEOUT in the device error word and the kernel returns normally:
 * no trap, no fault, the context stays usable. mf_get_device_error() then
 * reports MF_ERR_TIMEOUT. MF_ERR_INVALID_ARG for a limit out of range.
 */
mf_status mf_selftest_timeout(int64_t limit_ns, void* stream);

/*
 * Synchronises `stream`, then returns and clears the error the kernels
 * recorded on the current device since the last call (MF_OK if none,
 * MF_ERR_TIMEOUT if a pipeline wait ran out of time and the kernel gave up,
 * MF_ERR_BOUNDS from the checked build's range checks).
 */
mf_status mf_get_device_error(void* stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* MF_ATTN_H */
