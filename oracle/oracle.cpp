// Oracle: plain, slow, fp64 CPU implementation of the packed joint text+image
// attention forward of Mage-Flow's Native-Resolution MMDiT.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link,
// load or call this file: only the tests, the smoke check and the benchmark's
// CPU-baseline leg use it. It shares no code, header, table or helper with the
// CUDA library; the two are fed from the same seeded inputs and nothing else.
//
// What it computes, and where each step comes from:
//
// * Packing. Samples are flattened to token sequences of variable length and
//   concatenated without padding; sample i occupies tokens [s_i, s_i + L_i)
//   of the pack, s_i being the prefix sum of the lengths (per-sample
//   cumulative offsets). [Mage-Flow summary, "Native-Resolution MMDiT
//   (NR-MMDiT)": native-resolution packing; video overview, 00:03:16-00:04:03]
//   Within a sample the text tokens come first, then each latent grid of
//   H x W tokens flattened row-major; L_i = n_text + frames * H * W.
// * Modality-specific normalisation of the attention inputs. [summary,
//   "Native-Resolution MMDiT": modality-specific normalization; video
//   overview, 00:00:00]. Reading adopted (the pages do not give its form):
//   RMSNorm over head_dim per (token, head),
//       x_hat = x / sqrt(mean_m x_m^2 + eps) * gamma,
//   with one gamma vector of length head_dim per (q or k) x (text or image).
//   V is not normalised.
// * Per-sample 2D RoPE on image tokens. [video overview, 00:03:16; capabilities
//   page, "Key Capabilities": per-sample 2D RoPE preserving the native layout].
//   Reading adopted: a token at grid row r, column c (from 0, top-left origin)
//   rotates the first head_dim/2 dimensions by r and the last head_dim/2 by c,
//   in adjacent pairs (2j, 2j+1), pair j turning by pos * theta_j with
//   theta_j = 10000^(-2j/(head_dim/2)), (a, b) -> (a cos - b sin, a sin + b cos).
//   Text tokens are not rotated. Norm first, then rotation. Every frame of a
//   multi-grid sample (an editing target and its reference image) uses the
//   same grid positions.
// * 3D RoPE with a frame axis, for editing samples whose source latents are
//   concatenated with the target latents [summary, "Native-Resolution MMDiT",
//   Conditioning: a 3D RoPE whose frame dimension tells source from target].
//   Reading adopted (the pages give no split of head_dim): with frame_dims =
//   F > 0, dims [0, F) rotate by the frame index f (the sample's grids counted
//   from 0), dims [F, F + S) by r and dims [F + S, d) by c, S = (d - F) / 2;
//   each part pairs its own dims (first + 2j, first + 2j + 1) and turns pair j
//   by pos * 10000^(-2j / width), width being the part's size. F = 0 is the
//   2D rotation above (parts of width d/2 for r and c).
// * Joint self-attention confined to each sample [summary, "Native-Resolution
//   MMDiT": FlashAttention with per-sample cumulative offsets]: for query t in
//   sample i, s_u = (q_hat_t . k_hat_u) * scale over u in [s_i, s_i + L_i),
//   then o_t = sum_u exp(s_u - max s) v_u / sum_u exp(s_u - max s). Non-causal.
//   Computed in two passes (scores, then max, then the weighted sum): no
//   online rescaling.
// * Gradients of all of the above for training (oracle_attn_grad, at the end
//   of the file): the chain rule written out, on fp64 inputs.
//
// Inputs are bf16 bit patterns converted exactly to fp64; gammas are fp32
// values; all arithmetic is fp64.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

struct Segment {
  int64_t start;
  int64_t len;
  int64_t n_text;
  int64_t grid_h;
  int64_t grid_w;
  int64_t frames;
};

double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Lengths and starting offsets of every sample; false on an invalid sample.
bool make_segments(int n, const int32_t* n_text, const int32_t* grid_h, const int32_t* grid_w,
                   const int32_t* frames, std::vector<Segment>& segs, int64_t& total) {
  if (n < 0 || (n > 0 && (!n_text || !grid_h || !grid_w))) return false;
  segs.clear();
  total = 0;
  for (int i = 0; i < n; ++i) {
    Segment s;
    s.n_text = n_text[i];
    s.grid_h = grid_h[i];
    s.grid_w = grid_w[i];
    s.frames = frames ? frames[i] : 1;
    if (s.n_text < 0 || s.grid_h < 1 || s.grid_w < 1 || s.frames < 1) return false;
    s.len = s.n_text + s.frames * s.grid_h * s.grid_w;
    s.start = total;
    total += s.len;
    segs.push_back(s);
  }
  return true;
}

// Index of the sample that holds token t (starts are increasing).
size_t segment_of(const std::vector<Segment>& segs, int64_t t) {
  size_t lo = 0, hi = segs.size();
  while (hi - lo > 1) {
    size_t mid = (lo + hi) / 2;
    if (segs[mid].start <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// Modality, frame and grid position of token t of segment s.
void token_position(const Segment& s, int64_t t, bool& is_text, int64_t& f, int64_t& r,
                    int64_t& c) {
  int64_t j = t - s.start;
  if (j < s.n_text) {
    is_text = true;
    f = r = c = 0;
    return;
  }
  int64_t p = j - s.n_text;
  f = p / (s.grid_h * s.grid_w);
  int64_t in_frame = p % (s.grid_h * s.grid_w);  // every frame shares the grid positions
  r = in_frame / s.grid_w;
  c = in_frame % s.grid_w;
  is_text = false;
}

bool valid_frame_dims(int d, int frame_dims) {
  return frame_dims >= 0 && frame_dims % 4 == 0 && frame_dims <= d - 4;
}

// Rotation of an image token's vector in place: consecutive parts of head_dim
// for the frame (frame_dims wide, possibly empty), the grid row and the grid
// column; pair j of a part of width w turns by pos * 10000^(-2j/w). sign = -1
// applies the inverse (transposed) rotation.
void rotate_pairs(double* v, int d, int frame_dims, int64_t f, int64_t r, int64_t c, double sign) {
  const int spatial = (d - frame_dims) / 2;
  const int first[3] = {0, frame_dims, frame_dims + spatial};
  const int width[3] = {frame_dims, spatial, spatial};
  const int64_t pos[3] = {f, r, c};
  for (int axis = 0; axis < 3; ++axis) {
    for (int j = 0; j < width[axis] / 2; ++j) {
      double theta = std::pow(10000.0, -2.0 * j / width[axis]);
      double phi = sign * static_cast<double>(pos[axis]) * theta;
      double cs = std::cos(phi), sn = std::sin(phi);
      int i0 = first[axis] + 2 * j;
      double a = v[i0], b = v[i0 + 1];
      v[i0] = a * cs - b * sn;
      v[i0 + 1] = a * sn + b * cs;
    }
  }
}

// RMSNorm with the modality's gamma, then the rotation for image tokens:
// consecutive parts of head_dim for the frame (frame_dims wide, possibly
// empty), the grid row and the grid column.
void norm_rotate(const uint16_t* x, int d, const float* gamma, bool is_text, int64_t f, int64_t r,
                 int64_t c, int frame_dims, double eps, double* out) {
  double sum_sq = 0.0;
  for (int m = 0; m < d; ++m) {
    double v = bf16_value(x[m]);
    sum_sq += v * v;
  }
  double inv_rms = 1.0 / std::sqrt(sum_sq / d + eps);
  for (int m = 0; m < d; ++m) out[m] = bf16_value(x[m]) * inv_rms * static_cast<double>(gamma[m]);
  if (is_text) return;
  rotate_pairs(out, d, frame_dims, f, r, c, 1.0);
}

int resolve_threads(int n_threads) {
  if (n_threads > 0) return n_threads;
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

struct Job {
  size_t seg;
  int head;
  std::vector<int64_t> out_index;  // positions in the output array
  std::vector<int64_t> tokens;     // query tokens, same order
};

}  // namespace

extern "C" {

int oracle_abi_version() { return 2; }

// Total tokens of the pack, or -1 if a sample is invalid.
int64_t oracle_total_tokens(int n, const int32_t* n_text, const int32_t* grid_h,
                            const int32_t* grid_w, const int32_t* frames) {
  std::vector<Segment> segs;
  int64_t total = 0;
  if (!make_segments(n, n_text, grid_h, grid_w, frames, segs, total)) return -1;
  return total;
}

// Normalised and rotated q or k: x bf16 bits [T, heads, d] -> out fp64 [T, heads, d].
int oracle_qk_prologue(const uint16_t* x, int64_t total_tokens, int heads, int d,
                       const float* g_text, const float* g_img, int n, const int32_t* n_text,
                       const int32_t* grid_h, const int32_t* grid_w, const int32_t* frames,
                       double eps, int frame_dims, double* out) {
  std::vector<Segment> segs;
  int64_t total = 0;
  if (!make_segments(n, n_text, grid_h, grid_w, frames, segs, total)) return -1;
  if (total != total_tokens || heads < 1 || d < 4 || d % 4 != 0) return -1;
  if (!valid_frame_dims(d, frame_dims)) return -1;
  for (int64_t t = 0; t < total; ++t) {
    const Segment& s = segs[segment_of(segs, t)];
    bool is_text;
    int64_t f, r, c;
    token_position(s, t, is_text, f, r, c);
    for (int h = 0; h < heads; ++h) {
      int64_t row = t * heads + h;
      norm_rotate(x + row * d, d, is_text ? g_text : g_img, is_text, f, r, c, frame_dims, eps,
                  out + row * d);
    }
  }
  return 0;
}

// Attention output for selected (token, head) rows.
// rows[i] = token * heads + head; rows == NULL selects every row in order.
// out: fp64 [n_rows, d].
int oracle_joint_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const float* gq_text, const float* gq_img, const float* gk_text,
                      const float* gk_img, int n, const int32_t* n_text, const int32_t* grid_h,
                      const int32_t* grid_w, const int32_t* frames, int heads, int d, double eps,
                      int frame_dims, double scale, int64_t n_rows, const int64_t* rows,
                      double* out, int n_threads) {
  std::vector<Segment> segs;
  int64_t total = 0;
  if (!make_segments(n, n_text, grid_h, grid_w, frames, segs, total)) return -1;
  if (heads < 1 || d < 4 || d % 4 != 0) return -1;
  if (!valid_frame_dims(d, frame_dims)) return -1;
  if (!rows) n_rows = total * heads;
  if (n_rows < 0) return -1;

  // Group the requested rows by (segment, head), in blocks of at most 64 rows.
  std::vector<std::vector<std::pair<int64_t, int64_t>>> by_pair(segs.size() * heads);
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t row = rows ? rows[i] : i;
    if (row < 0 || row >= total * heads) return -1;
    int64_t t = row / heads;
    int h = static_cast<int>(row % heads);
    size_t si = segment_of(segs, t);
    by_pair[si * heads + h].push_back({t, i});
  }
  std::vector<Job> jobs;
  for (size_t pi = 0; pi < by_pair.size(); ++pi) {
    auto& lst = by_pair[pi];
    for (size_t b = 0; b < lst.size(); b += 64) {
      Job job;
      job.seg = pi / heads;
      job.head = static_cast<int>(pi % heads);
      for (size_t e = b; e < std::min(lst.size(), b + 64); ++e) {
        job.tokens.push_back(lst[e].first);
        job.out_index.push_back(lst[e].second);
      }
      jobs.push_back(std::move(job));
    }
  }
  // Longest segments first, so the threads finish together.
  std::stable_sort(jobs.begin(), jobs.end(), [&](const Job& a, const Job& b) {
    return segs[a.seg].len > segs[b.seg].len;
  });

  std::atomic<size_t> next{0};
  auto worker = [&]() {
    std::vector<double> k_hat, v_val, q_hat(d), scores, acc(d);
    for (;;) {
      size_t ji = next.fetch_add(1);
      if (ji >= jobs.size()) break;
      const Job& job = jobs[ji];
      const Segment& s = segs[job.seg];
      const int h = job.head;
      k_hat.assign(static_cast<size_t>(s.len) * d, 0.0);
      v_val.assign(static_cast<size_t>(s.len) * d, 0.0);
      scores.assign(static_cast<size_t>(s.len), 0.0);
      for (int64_t u = 0; u < s.len; ++u) {
        int64_t t = s.start + u;
        bool is_text;
        int64_t f, r, c;
        token_position(s, t, is_text, f, r, c);
        int64_t row = t * heads + h;
        norm_rotate(k + row * d, d, is_text ? gk_text : gk_img, is_text, f, r, c, frame_dims, eps,
                    &k_hat[static_cast<size_t>(u) * d]);
        for (int m = 0; m < d; ++m) v_val[static_cast<size_t>(u) * d + m] = bf16_value(v[row * d + m]);
      }
      for (size_t qi = 0; qi < job.tokens.size(); ++qi) {
        int64_t t = job.tokens[qi];
        bool is_text;
        int64_t f, r, c;
        token_position(s, t, is_text, f, r, c);
        norm_rotate(q + (t * heads + h) * d, d, is_text ? gq_text : gq_img, is_text, f, r, c,
                    frame_dims, eps, q_hat.data());
        // Pass 1: scores and their maximum.
        double mx = -std::numeric_limits<double>::infinity();
        for (int64_t u = 0; u < s.len; ++u) {
          double dot = 0.0;
          const double* kr = &k_hat[static_cast<size_t>(u) * d];
          for (int m = 0; m < d; ++m) dot += q_hat[m] * kr[m];
          scores[u] = dot * scale;
          mx = std::max(mx, scores[u]);
        }
        // Pass 2: weights and the weighted sum of values.
        double denom = 0.0;
        std::fill(acc.begin(), acc.end(), 0.0);
        for (int64_t u = 0; u < s.len; ++u) {
          double w = std::exp(scores[u] - mx);
          denom += w;
          const double* vr = &v_val[static_cast<size_t>(u) * d];
          for (int m = 0; m < d; ++m) acc[m] += w * vr[m];
        }
        double* o = out + job.out_index[qi] * d;
        for (int m = 0; m < d; ++m) o[m] = acc[m] / denom;
      }
    }
  };
  int nt = std::min<int>(resolve_threads(n_threads), std::max<size_t>(jobs.size(), 1));
  std::vector<std::thread> pool;
  for (int i = 1; i < nt; ++i) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  return 0;
}

// Brute force for small packs: for every head, the full T x T score matrix
// over the whole pack, entries between different samples set to -inf, and a
// row softmax over all T columns. Token positions are enumerated by nested
// loops over samples, frames, rows and columns instead of being decoded.
// out: fp64 [T, heads, d].
int oracle_dense_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const float* gq_text, const float* gq_img, const float* gk_text,
                      const float* gk_img, int n, const int32_t* n_text, const int32_t* grid_h,
                      const int32_t* grid_w, const int32_t* frames, int heads, int d, double eps,
                      int frame_dims, double scale, double* out) {
  if (n < 1 || heads < 1 || d < 4 || d % 4 != 0) return -1;
  if (!valid_frame_dims(d, frame_dims)) return -1;
  std::vector<int> sample_id;
  std::vector<int> text_flag;
  std::vector<int64_t> pos_f, pos_r, pos_c;
  for (int i = 0; i < n; ++i) {
    int f_count = frames ? frames[i] : 1;
    if (n_text[i] < 0 || grid_h[i] < 1 || grid_w[i] < 1 || f_count < 1) return -1;
    for (int j = 0; j < n_text[i]; ++j) {
      sample_id.push_back(i);
      text_flag.push_back(1);
      pos_f.push_back(0);
      pos_r.push_back(0);
      pos_c.push_back(0);
    }
    for (int f = 0; f < f_count; ++f)
      for (int r = 0; r < grid_h[i]; ++r)
        for (int c = 0; c < grid_w[i]; ++c) {
          sample_id.push_back(i);
          text_flag.push_back(0);
          pos_f.push_back(f);
          pos_r.push_back(r);
          pos_c.push_back(c);
        }
  }
  const int64_t T = static_cast<int64_t>(sample_id.size());
  std::vector<double> qh(static_cast<size_t>(T) * d), kh(static_cast<size_t>(T) * d);
  std::vector<double> s(static_cast<size_t>(T) * T);
  for (int h = 0; h < heads; ++h) {
    for (int64_t t = 0; t < T; ++t) {
      int64_t row = t * heads + h;
      bool txt = text_flag[t] != 0;
      norm_rotate(q + row * d, d, txt ? gq_text : gq_img, txt, pos_f[t], pos_r[t], pos_c[t],
                  frame_dims, eps, &qh[static_cast<size_t>(t) * d]);
      norm_rotate(k + row * d, d, txt ? gk_text : gk_img, txt, pos_f[t], pos_r[t], pos_c[t],
                  frame_dims, eps, &kh[static_cast<size_t>(t) * d]);
    }
    for (int64_t t = 0; t < T; ++t)
      for (int64_t u = 0; u < T; ++u) {
        double val = -std::numeric_limits<double>::infinity();
        if (sample_id[t] == sample_id[u]) {
          double dot = 0.0;
          for (int m = 0; m < d; ++m)
            dot += qh[static_cast<size_t>(t) * d + m] * kh[static_cast<size_t>(u) * d + m];
          val = dot * scale;
        }
        s[static_cast<size_t>(t) * T + u] = val;
      }
    for (int64_t t = 0; t < T; ++t) {
      double* srow = &s[static_cast<size_t>(t) * T];
      double mx = *std::max_element(srow, srow + T);
      double denom = 0.0;
      for (int64_t u = 0; u < T; ++u) {
        srow[u] = std::exp(srow[u] - mx);
        denom += srow[u];
      }
      double* o = out + (t * heads + h) * d;
      for (int m = 0; m < d; ++m) {
        double a = 0.0;
        for (int64_t u = 0; u < T; ++u) a += srow[u] * bf16_value(v[(u * heads + h) * d + m]);
        o[m] = a / denom;
      }
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Gradients, for training. The pages' headline speedup is for training the
// NR-MMDiT [video overview, 00:05:08; summary, "Training Infrastructure"], so
// the path's backward is the derivative of the forward above, by the chain
// rule, for a loss L with dL/dout = G:
//   P_tu = exp(s_tu - M_t) / Z_t, s_tu = scale * q_hat_t . k_hat_u   (within a sample)
//   dv_u     = sum_t P_tu G_t
//   dP_tu    = G_t . v_u,  D_t = sum_u P_tu dP_tu,  dS_tu = P_tu (dP_tu - D_t)
//   dq_hat_t = scale * sum_u dS_tu k_hat_u,  dk_hat_u = scale * sum_t dS_tu q_hat_t
//   dy       = R(pos)^T dx_hat                      (rotation transposed; text: dy = dx_hat)
//   dgamma  += dy * x_n                              (per role and modality, summed over tokens and heads)
//   dx       = r * (dx_n - x_n * (x_n . dx_n) / d),  dx_n = dy * gamma
// with x_n = x * r, r = 1 / sqrt(mean(x^2) + eps). Inputs here are fp64 (so
// finite differences can probe them); the bf16 forward above is the same
// function of the same values.
// ---------------------------------------------------------------------------

namespace {

struct GradJob {
  size_t seg;
  int head;
  int64_t lo, hi;  // rows of the sample (query rows or key rows), relative to its start
};

}  // namespace

int oracle_attn_grad(const double* q, const double* k, const double* v, const double* gq_text,
                     const double* gq_img, const double* gk_text, const double* gk_img,
                     const double* dout, int n, const int32_t* n_text, const int32_t* grid_h,
                     const int32_t* grid_w, const int32_t* frames, int heads, int d, double eps,
                     int frame_dims, double scale, double* out, double* lse, double* dq,
                     double* dk, double* dv, double* dgamma, int n_threads) {
  std::vector<Segment> segs;
  int64_t total = 0;
  if (!make_segments(n, n_text, grid_h, grid_w, frames, segs, total)) return -1;
  if (heads < 1 || d < 4 || d % 4 != 0 || !valid_frame_dims(d, frame_dims)) return -1;
  if (dout && (!dq || !dk || !dv || !dgamma)) return -1;
  const size_t rows = static_cast<size_t>(total) * heads;

  // Per (token, head) of q and k: r, x_n and the rotated x_hat.
  std::vector<double> rq(rows), rk(rows), qn(rows * d), kn(rows * d), qh(rows * d), kh(rows * d);
  std::vector<int64_t> pf(total), pr(total), pc(total);
  std::vector<char> txt(total);
  for (int64_t t = 0; t < total; ++t) {
    bool is_text;
    token_position(segs[segment_of(segs, t)], t, is_text, pf[t], pr[t], pc[t]);
    txt[t] = is_text;
    for (int h = 0; h < heads; ++h) {
      const size_t row = static_cast<size_t>(t) * heads + h;
      for (int which = 0; which < 2; ++which) {
        const double* x = (which == 0 ? q : k) + row * d;
        const double* g = which == 0 ? (is_text ? gq_text : gq_img) : (is_text ? gk_text : gk_img);
        double sum_sq = 0.0;
        for (int m = 0; m < d; ++m) sum_sq += x[m] * x[m];
        const double r = 1.0 / std::sqrt(sum_sq / d + eps);
        double* xn = (which == 0 ? qn : kn).data() + row * d;
        double* xh = (which == 0 ? qh : kh).data() + row * d;
        for (int m = 0; m < d; ++m) {
          xn[m] = x[m] * r;
          xh[m] = xn[m] * g[m];
        }
        if (!is_text) rotate_pairs(xh, d, frame_dims, pf[t], pr[t], pc[t], 1.0);
        (which == 0 ? rq : rk)[row] = r;
      }
    }
  }

  auto score = [&](size_t row_q, size_t row_k) {
    double dot = 0.0;
    for (int m = 0; m < d; ++m) dot += qh[row_q * d + m] * kh[row_k * d + m];
    return dot * scale;
  };
  auto run_jobs = [&](const std::vector<GradJob>& jobs, auto&& body) {
    std::atomic<size_t> next{0};
    auto worker = [&]() {
      for (;;) {
        size_t ji = next.fetch_add(1);
        if (ji >= jobs.size()) break;
        body(jobs[ji]);
      }
    };
    int nt = std::min<int>(resolve_threads(n_threads), std::max<size_t>(jobs.size(), 1));
    std::vector<std::thread> pool;
    for (int i = 1; i < nt; ++i) pool.emplace_back(worker);
    worker();
    for (auto& th : pool) th.join();
  };
  std::vector<GradJob> jobs;
  for (size_t si = 0; si < segs.size(); ++si)
    for (int h = 0; h < heads; ++h)
      for (int64_t lo = 0; lo < segs[si].len; lo += 64)
        jobs.push_back({si, h, lo, std::min<int64_t>(segs[si].len, lo + 64)});

  // Pass 1, per query row: M_t, Z_t, the output and (with a gradient) D_t.
  std::vector<double> M(rows), Z(rows), D(rows, 0.0), o(rows * d);
  run_jobs(jobs, [&](const GradJob& jb) {
    const Segment& s = segs[jb.seg];
    std::vector<double> sc(static_cast<size_t>(s.len));
    for (int64_t i = jb.lo; i < jb.hi; ++i) {
      const size_t rt = static_cast<size_t>(s.start + i) * heads + jb.head;
      double mx = -std::numeric_limits<double>::infinity();
      for (int64_t u = 0; u < s.len; ++u) {
        sc[u] = score(rt, static_cast<size_t>(s.start + u) * heads + jb.head);
        mx = std::max(mx, sc[u]);
      }
      double z = 0.0;
      for (int64_t u = 0; u < s.len; ++u) z += std::exp(sc[u] - mx);
      M[rt] = mx;
      Z[rt] = z;
      double* ot = &o[rt * d];
      for (int m = 0; m < d; ++m) ot[m] = 0.0;
      double dsum = 0.0;
      for (int64_t u = 0; u < s.len; ++u) {
        const size_t ru = static_cast<size_t>(s.start + u) * heads + jb.head;
        const double p = std::exp(sc[u] - mx) / z;
        for (int m = 0; m < d; ++m) ot[m] += p * v[ru * d + m];
        if (dout) {
          double dp = 0.0;
          for (int m = 0; m < d; ++m) dp += dout[rt * d + m] * v[ru * d + m];
          dsum += p * dp;
        }
      }
      D[rt] = dsum;
    }
  });
  if (out) std::copy(o.begin(), o.end(), out);
  if (lse)  // log of the softmax normaliser: log sum_u exp(s_tu) = M_t + log Z_t, [T, heads]
    for (size_t r = 0; r < rows; ++r) lse[r] = M[r] + std::log(Z[r]);
  if (!dout) return 0;

  // P_tu and dS_tu from the stored row statistics.
  auto p_ds = [&](size_t rt, size_t ru, double& p, double& ds) {
    p = std::exp(score(rt, ru) - M[rt]) / Z[rt];
    double dp = 0.0;
    for (int m = 0; m < d; ++m) dp += dout[rt * d + m] * v[ru * d + m];
    ds = p * (dp - D[rt]);
  };
  // Pass 2, per query row: dq_hat.  Pass 3, per key row: dk_hat and dv.
  std::vector<double> dqh(rows * d, 0.0), dkh(rows * d, 0.0);
  run_jobs(jobs, [&](const GradJob& jb) {
    const Segment& s = segs[jb.seg];
    for (int64_t i = jb.lo; i < jb.hi; ++i) {
      const size_t rt = static_cast<size_t>(s.start + i) * heads + jb.head;
      double* acc = &dqh[rt * d];
      for (int64_t u = 0; u < s.len; ++u) {
        const size_t ru = static_cast<size_t>(s.start + u) * heads + jb.head;
        double p, ds;
        p_ds(rt, ru, p, ds);
        for (int m = 0; m < d; ++m) acc[m] += scale * ds * kh[ru * d + m];
      }
    }
  });
  run_jobs(jobs, [&](const GradJob& jb) {
    const Segment& s = segs[jb.seg];
    for (int64_t i = jb.lo; i < jb.hi; ++i) {
      const size_t ru = static_cast<size_t>(s.start + i) * heads + jb.head;
      double* acc_k = &dkh[ru * d];
      double* acc_v = dv + ru * d;
      for (int m = 0; m < d; ++m) acc_v[m] = 0.0;
      for (int64_t t = 0; t < s.len; ++t) {
        const size_t rt = static_cast<size_t>(s.start + t) * heads + jb.head;
        double p, ds;
        p_ds(rt, ru, p, ds);
        for (int m = 0; m < d; ++m) {
          acc_k[m] += scale * ds * qh[rt * d + m];
          acc_v[m] += p * dout[rt * d + m];
        }
      }
    }
  });

  // Back through the rotation and the norm; gammas summed in token order.
  for (int i = 0; i < 4 * d; ++i) dgamma[i] = 0.0;
  std::vector<double> dy(d);
  for (int64_t t = 0; t < total; ++t) {
    for (int h = 0; h < heads; ++h) {
      const size_t row = static_cast<size_t>(t) * heads + h;
      for (int which = 0; which < 2; ++which) {
        const double* dxh = (which == 0 ? dqh : dkh).data() + row * d;
        const double* xn = (which == 0 ? qn : kn).data() + row * d;
        const double* g = which == 0 ? (txt[t] ? gq_text : gq_img) : (txt[t] ? gk_text : gk_img);
        const double r = (which == 0 ? rq : rk)[row];
        double* dg = dgamma + (2 * which + (txt[t] ? 0 : 1)) * d;
        double* dx = (which == 0 ? dq : dk) + row * d;
        for (int m = 0; m < d; ++m) dy[m] = dxh[m];
        if (!txt[t]) rotate_pairs(dy.data(), d, frame_dims, pf[t], pr[t], pc[t], -1.0);
        double dot = 0.0;
        for (int m = 0; m < d; ++m) {
          dg[m] += dy[m] * xn[m];
          dot += xn[m] * (dy[m] * g[m]);
        }
        for (int m = 0; m < d; ++m) dx[m] = r * (dy[m] * g[m] - xn[m] * dot / d);
      }
    }
  }
  return 0;
}

}  // extern "C"
