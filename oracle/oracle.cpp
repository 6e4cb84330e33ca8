// oracle.cpp — plain, slow, fp64 CPU oracle of 3D block-sparse attention.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline / reference legs of bench.py may load or call this code.  The
// product path (libbsa and its Python binding) never touches it, and this file
// shares no code, header, table or constant with the CUDA implementation.
//
// What it computes is the head-wise sparse attention executor of
//   SPADE: An Input-Adaptive Sparse Attention Engine for Fast Video Diffusion
//   Models Inference, §3.3 "Head-wise Sparse Attention":
//     blocked layout -> one mean summary per Q/K block -> inter-block
//     importance matrix -> Top-K / Top-P -> block-sparse attention (§2.2,
//     Eq. (2)) -> output restored to the original layout,
// with the block-shape convention of the DecoupAttn Plans README ("Contents":
// frames x rows x cols of one key block) and the density of the blog "Does
// sparse attention actually speed up video generation?" ("How this was
// measured": the fraction of key blocks each query block keeps).
//
// Every quantity is computed by its plain definition in double precision,
// one element at a time, with no blocking, fusion or reordering.  Inputs are
// float arrays (bf16 inputs are widened to float exactly by the caller).
//
// Readings of points the pages leave open (each one is listed in the design
// notes of the repository):
//   R1 token order: video token (t,y,x) at n = (t*H + y)*W + x (SPADE §2.1,
//      the latent is flattened to a 1D sequence); text tokens follow.
//   R2 block order (tb,yb,xb) raster; slot order (dt,dy,dx) raster; the grid
//      is padded at the high end of each axis; pad slots are 0, are never
//      keys and give output 0 as queries.
//   R3 centroid = arithmetic mean over the valid tokens of a block.
//   R4 inter-block score s_ij = qbar_i . kbar_j / sqrt(D), p_i = softmax_j(s_i)
//      over the nb video key blocks.
//   R5 k = ceil(rho * nb - 1e-9) clamped to [1, nb].
//   R6 order for selection: p descending, then key-block id ascending.
//   R7 Top-P: the smallest m >= 1 whose descending prefix mass reaches tau.
//   R8 text blocks are not scored; every video query block also attends all
//      text key blocks; text query tokens attend every token.
//   R9 lists are stored in ascending block id, text blocks last.
//   R15 SICS: a zero vector has no direction and contributes nothing.
//   R18 local window: key blocks j with i - left <= j <= i + right over the
//       block sequence; a negative side is unbounded; (-1, -1) = no window.
//   R19 attention sink: the key blocks holding any of the first S tokens of
//       the original sequence.
//   R20 intra scores: one per key block, broadcast to every query block of
//       the head; selected by the Top-K / Top-P rule on the scores.
//   R21 DSA / DSA2 inter-estimators: the largest q . k over the summaries'
//       boxes (DSA: query fixed at the box centre).  Parity unpinned: the
//       pages give the summaries but not the estimator equations, so
//       orc_scores_box is checked against this reading (a brute force over
//       the box corners), not against a value or formula of the pages.
//
// Geometry array g[10] = {B, T, H, W, bf, br, bc, Hd, D, n_text}.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

namespace {

struct Geom {
  long long B, T, H, W, bf, br, bc, Hd, D, n_text;
  long long nbt, nby, nbx, nb, bs, nb_text, n_video, n_tot, npad_tot;
};

Geom make_geom(const int* g) {
  Geom G;
  G.B = g[0]; G.T = g[1]; G.H = g[2]; G.W = g[3];
  G.bf = g[4]; G.br = g[5]; G.bc = g[6]; G.Hd = g[7]; G.D = g[8];
  G.n_text = g[9];
  G.nbt = (G.T + G.bf - 1) / G.bf;
  G.nby = (G.H + G.br - 1) / G.br;
  G.nbx = (G.W + G.bc - 1) / G.bc;
  G.nb = G.nbt * G.nby * G.nbx;
  G.bs = G.bf * G.br * G.bc;
  G.nb_text = (G.n_text + G.bs - 1) / G.bs;
  G.n_video = G.T * G.H * G.W;
  G.n_tot = G.n_video + G.n_text;
  G.npad_tot = (G.nb + G.nb_text) * G.bs;
  return G;
}

int n_threads() {
  const char* e = std::getenv("ORACLE_THREADS");
  if (e && std::atoi(e) > 0) return std::atoi(e);
  unsigned h = std::thread::hardware_concurrency();
  return h ? (int)h : 1;
}

// Runs f(i) for i in [0, n) on all threads, static interleaved split.
template <class F>
void parallel_for(long long n, F f) {
  int nt = n_threads();
  if (nt > n) nt = (int)std::max<long long>(n, 1);
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([=, &f] {
      for (long long i = t; i < n; i += nt) f(i);
    });
  for (auto& th : pool) th.join();
}

// Block id and slot of a video token (t, y, x): read R2 in the token -> slot
// direction.
void video_slot(const Geom& G, long long t, long long y, long long x,
                long long* blk, long long* slot) {
  long long tb = t / G.bf, dt = t % G.bf;
  long long yb = y / G.br, dy = y % G.br;
  long long xb = x / G.bc, dx = x % G.bc;
  *blk = (tb * G.nby + yb) * G.nbx + xb;
  *slot = (dt * G.br + dy) * G.bc + dx;
}

// Original token index of every valid token of block j (video or text).
std::vector<long long> block_tokens(const Geom& G, long long j) {
  std::vector<long long> out;
  if (j < G.nb) {
    long long tb = j / (G.nby * G.nbx);
    long long yb = (j / G.nbx) % G.nby;
    long long xb = j % G.nbx;
    for (long long dt = 0; dt < G.bf; ++dt)
      for (long long dy = 0; dy < G.br; ++dy)
        for (long long dx = 0; dx < G.bc; ++dx) {
          long long t = tb * G.bf + dt, y = yb * G.br + dy, x = xb * G.bc + dx;
          if (t < G.T && y < G.H && x < G.W) out.push_back((t * G.H + y) * G.W + x);
        }
  } else {
    long long u0 = (j - G.nb) * G.bs;
    for (long long u = u0; u < u0 + G.bs && u < G.n_text; ++u)
      out.push_back(G.n_video + u);
  }
  return out;
}

// Top-K / Top-P rule over one row of nonnegative weights v[0..nb) (R5-R7,
// R12): order by v descending, then index ascending; Top-K keeps
// k_for_density(param) entries, Top-P the smallest m >= 1 whose prefix sum
// reaches param * total.  `chosen` gets the kept indices; `tie` is set when
// the cut sits on a near-tie (1e-5 relative).
int k_for_density_(double rho, long long nb) {
  long long k = (long long)std::ceil(rho * (double)nb - 1e-9);
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return (int)k;
}

void select_rule(const double* v, long long nb, int mode, double param, double total,
                 std::vector<long long>& chosen, int& tie) {
  std::vector<long long> order(nb);
  for (long long j = 0; j < nb; ++j) order[j] = j;
  std::sort(order.begin(), order.end(), [&](long long a, long long b) {
    if (v[a] != v[b]) return v[a] > v[b];
    return a < b;
  });
  long long m;
  if (mode == 0) {
    m = k_for_density_(param, nb);
    if (m < nb) {
      double a = v[order[m - 1]], b = v[order[m]];
      if (std::fabs(a - b) <= 1e-5 * std::fabs(a)) tie = 1;
    }
  } else {
    const double target = param * total;
    double cum = 0.0, before = 0.0;
    m = 0;
    while (m < nb) {
      before = cum;
      cum += v[order[m]];
      ++m;
      if (cum >= target) break;
    }
    if (std::fabs(before - target) <= 1e-5 * target) tie = 1;
    if (std::fabs(cum - target) <= 1e-5 * target) tie = 1;
    if (m < nb) {
      double a = v[order[m - 1]], b = v[order[m]];
      if (std::fabs(a - b) <= 1e-5 * std::fabs(a)) tie = 1;
    }
  }
  chosen.assign(order.begin(), order.begin() + m);
}

}  // namespace

extern "C" {

int orc_threads(void) { return n_threads(); }

// Layout transform (SPADE §3.3: Q, K, V "rearranged into a blocked layout").
// x [B, Ntot, Hd, D] -> x_blk [B, Hd, Npad_tot, D]; pad slots are 0 (R2).
void orc_permute(const int* g, const float* x, double* x_blk) {
  Geom G = make_geom(g);
  std::memset(x_blk, 0, sizeof(double) * G.B * G.Hd * G.npad_tot * G.D);
  for (long long b = 0; b < G.B; ++b)
    for (long long n = 0; n < G.n_tot; ++n) {
      long long blk, slot;
      if (n < G.n_video) {
        long long t = n / (G.H * G.W), y = (n / G.W) % G.H, xx = n % G.W;
        video_slot(G, t, y, xx, &blk, &slot);
      } else {
        blk = G.nb + (n - G.n_video) / G.bs;
        slot = (n - G.n_video) % G.bs;
      }
      for (long long h = 0; h < G.Hd; ++h)
        for (long long d = 0; d < G.D; ++d)
          x_blk[((b * G.Hd + h) * G.npad_tot + blk * G.bs + slot) * G.D + d] =
              (double)x[((b * G.n_tot + n) * G.Hd + h) * G.D + d];
    }
}

// Inverse layout transform (SPADE §3.3: "output blocks are restored to the
// original layout"); pad slots are dropped.
void orc_unpermute(const int* g, const double* x_blk, double* x) {
  Geom G = make_geom(g);
  for (long long b = 0; b < G.B; ++b)
    for (long long n = 0; n < G.n_tot; ++n) {
      long long blk, slot;
      if (n < G.n_video) {
        long long t = n / (G.H * G.W), y = (n / G.W) % G.H, xx = n % G.W;
        video_slot(G, t, y, xx, &blk, &slot);
      } else {
        blk = G.nb + (n - G.n_video) / G.bs;
        slot = (n - G.n_video) % G.bs;
      }
      for (long long h = 0; h < G.Hd; ++h)
        for (long long d = 0; d < G.D; ++d)
          x[((b * G.n_tot + n) * G.Hd + h) * G.D + d] =
              x_blk[((b * G.Hd + h) * G.npad_tot + blk * G.bs + slot) * G.D + d];
    }
}

// Mean summarizer (SPADE §3.1 MEAN-SPADE, (q_mean, k_mean); §3.3 summaries
// Q', K' of shape (N_blocks, d_head)); R3: mean over valid tokens.
// x [B, Ntot, Hd, D] -> cent [B, Hd, nb, D].
void orc_centroids(const int* g, const float* x, double* cent) {
  Geom G = make_geom(g);
  std::vector<long long> count(G.nb, 0);
  std::memset(cent, 0, sizeof(double) * G.B * G.Hd * G.nb * G.D);
  for (long long n = 0; n < G.n_video; ++n) {
    long long t = n / (G.H * G.W), y = (n / G.W) % G.H, xx = n % G.W, blk, slot;
    video_slot(G, t, y, xx, &blk, &slot);
    count[blk] += 1;
    for (long long b = 0; b < G.B; ++b)
      for (long long h = 0; h < G.Hd; ++h)
        for (long long d = 0; d < G.D; ++d)
          cent[((b * G.Hd + h) * G.nb + blk) * G.D + d] +=
              (double)x[((b * G.n_tot + n) * G.Hd + h) * G.D + d];
  }
  for (long long b = 0; b < G.B; ++b)
    for (long long h = 0; h < G.Hd; ++h)
      for (long long blk = 0; blk < G.nb; ++blk)
        for (long long d = 0; d < G.D; ++d)
          cent[((b * G.Hd + h) * G.nb + blk) * G.D + d] /= (double)count[blk];
}

// Inter-block estimator (SPADE §3.1 "the dot product of blue vectors gives
// inter-block importance", §3.3 N_Qb x N_Kb matrix); R4:
// p[b,h,i,j] = softmax_j( qbar_i . kbar_j / sqrt(D) ).
void orc_scores(const int* g, const double* qc, const double* kc, double* p) {
  Geom G = make_geom(g);
  const double scale = 1.0 / std::sqrt((double)G.D);
  parallel_for(G.B * G.Hd * G.nb, [&](long long row) {
    long long bh = row / G.nb;
    const double* q = qc + row * G.D;
    double* out = p + row * G.nb;
    double m = -INFINITY;
    for (long long j = 0; j < G.nb; ++j) {
      const double* k = kc + (bh * G.nb + j) * G.D;
      double s = 0.0;
      for (long long d = 0; d < G.D; ++d) s += q[d] * k[d];
      out[j] = s * scale;
      m = std::max(m, out[j]);
    }
    double z = 0.0;
    for (long long j = 0; j < G.nb; ++j) {
      out[j] = std::exp(out[j] - m);
      z += out[j];
    }
    for (long long j = 0; j < G.nb; ++j) out[j] /= z;
  });
}

// Number of key blocks a density keeps (R5; the blog's "fraction of key
// blocks each query block keeps").
int orc_k_for_density(double rho, int nb) { return k_for_density_(rho, nb); }

// Top-K / Top-P selection (SPADE §3.1 "Top-K/Top-P mode"; §3.3 "Scores are
// filtered by Top-K or Top-P"; inter-top value = "Top-P cumulative threshold
// or Top-K keep").  mode 0 = top-k with params[h] = density, mode 1 = top-p
// with params[h] = tau.  Lists: ascending video ids then text ids (R8, R9).
// tie[row] = 1 where the decision is within the 1e-5 relative tolerance of
// flipping (R6/R7 boundary), else 0.
void orc_select(const int* g, const double* p, int mode, const double* params,
                int kmax, int* idx, int* cnt, int* tie) {
  Geom G = make_geom(g);
  parallel_for(G.B * G.Hd * G.nb, [&](long long row) {
    long long h = (row / G.nb) % G.Hd;
    std::vector<long long> chosen;
    int is_tie = 0;
    select_rule(p + row * G.nb, G.nb, mode, params[h], 1.0, chosen, is_tie);
    std::sort(chosen.begin(), chosen.end());
    int* out = idx + row * kmax;
    long long c = 0;
    for (long long j : chosen) out[c++] = (int)j;
    for (long long t = 0; t < G.nb_text; ++t) out[c++] = (int)(G.nb + t);
    cnt[row] = (int)c;
    tie[row] = is_tie;
  });
}

// Block lists of the mask union (SPADE §3.3: "intra scores are broadcast and
// OR-combined with inter scores.  The result is united with local-window and
// attention-sink masks"; §3.2 policy: local-window length, intra-top value,
// inter-top value; §3.1 attention-sink length).  Per video query block i of
// head h the list holds, in ascending id, the union of
//   inter:  the Top-K / Top-P selection of p[b,h,i,:] (as orc_select);
//   window: key blocks j with i - win_left <= j <= i + win_right (R18: a
//           sliding window over the block sequence, (left, right) as in
//           LongLive's window_size; a negative side is unbounded, and
//           (-1, -1) turns the window off);
//   sink:   key blocks holding any of the first sink_tokens tokens of the
//           original sequence (R19);
//   intra:  when intra != NULL and intra_params[h] > 0, the key blocks that
//           the same rule selects from the intra scores intra[b,h,:] (R20:
//           one score per key block, broadcast to every query block); Top-P
//           takes the shortest descending prefix whose sum reaches
//           tau * (sum of all scores);
// then the text key blocks.  tie[] flags rows whose inter selection, or
// whose head's intra selection, sits on a tie (R12).
void orc_select_union(const int* g, const double* p, int mode, const double* params, int kmax,
                      const double* intra, int intra_mode, const double* intra_params,
                      int win_left, int win_right, long long sink_tokens,
                      int* idx, int* cnt, int* tie) {
  Geom G = make_geom(g);
  std::vector<char> sink(G.nb, 0);
  for (long long j = 0; j < G.nb; ++j) {
    std::vector<long long> toks = block_tokens(G, j);
    for (long long t : toks)
      if (t < sink_tokens) sink[j] = 1;
  }
  std::vector<std::vector<char>> intra_set(G.B * G.Hd, std::vector<char>(G.nb, 0));
  std::vector<int> intra_tie(G.B * G.Hd, 0);
  if (intra != nullptr && intra_params != nullptr) {
    for (long long bh = 0; bh < G.B * G.Hd; ++bh) {
      const double prm = intra_params[bh % G.Hd];
      if (!(prm > 0.0)) continue;
      const double* v = intra + bh * G.nb;
      double total = 0.0;
      for (long long j = 0; j < G.nb; ++j) total += v[j];
      std::vector<long long> chosen;
      select_rule(v, G.nb, intra_mode, prm, total, chosen, intra_tie[bh]);
      for (long long j : chosen) intra_set[bh][j] = 1;
    }
  }
  const bool window = !(win_left < 0 && win_right < 0);
  parallel_for(G.B * G.Hd * G.nb, [&](long long row) {
    long long bh = row / G.nb, h = bh % G.Hd, i = row % G.nb;
    std::vector<long long> chosen;
    int is_tie = 0;
    select_rule(p + row * G.nb, G.nb, mode, params[h], 1.0, chosen, is_tie);
    std::vector<char> take(G.nb, 0);
    for (long long j : chosen) take[j] = 1;
    for (long long j = 0; j < G.nb; ++j) {
      if (window && (win_left < 0 || j >= i - win_left) && (win_right < 0 || j <= i + win_right))
        take[j] = 1;
      if (sink[j] || intra_set[bh][j]) take[j] = 1;
    }
    int* out = idx + row * kmax;
    long long c = 0;
    for (long long j = 0; j < G.nb; ++j)
      if (take[j]) out[c++] = (int)j;
    for (long long t = 0; t < G.nb_text; ++t) out[c++] = (int)(G.nb + t);
    cnt[row] = (int)c;
    tie[row] = is_tie | intra_tie[bh];
  });
}

// Block-sparse attention (SPADE §2.2, Eq. (2)): for each valid query token,
// softmax(q.k/sqrt(D)) over the union of the valid keys of its selected key
// blocks (M = 0 there, -inf elsewhere), applied to V; §2.2 Eq. (1) for text
// query tokens, which attend every token (R8).  Works on the ORIGINAL layout.
//   rows: NULL = every token (o is [B, Ntot, Hd, D]); otherwise n_rows token
//   indices, and o is [B, n_rows, Hd, D].
void orc_attention(const int* g, const float* q, const float* k, const float* v,
                   const int* idx, const int* cnt, int kmax,
                   const long long* rows, long long n_rows, double* o) {
  Geom G = make_geom(g);
  const double scale = 1.0 / std::sqrt((double)G.D);
  long long nr = rows ? n_rows : G.n_tot;
  parallel_for(G.B * G.Hd * nr, [&](long long task) {
    long long b = task / (G.Hd * nr);
    long long h = (task / nr) % G.Hd;
    long long r = task % nr;
    long long n = rows ? rows[r] : r;
    // The set of key tokens this query may attend.
    std::vector<long long> keys;
    if (n < G.n_video) {
      long long t = n / (G.H * G.W), y = (n / G.W) % G.H, xx = n % G.W, blk, slot;
      video_slot(G, t, y, xx, &blk, &slot);
      const int* list = idx + ((b * G.Hd + h) * G.nb + blk) * kmax;
      int c = cnt[(b * G.Hd + h) * G.nb + blk];
      for (int e = 0; e < c; ++e) {
        std::vector<long long> tk = block_tokens(G, list[e]);
        keys.insert(keys.end(), tk.begin(), tk.end());
      }
    } else {
      for (long long j = 0; j < G.nb + G.nb_text; ++j) {
        std::vector<long long> tk = block_tokens(G, j);
        keys.insert(keys.end(), tk.begin(), tk.end());
      }
    }
    const float* qv = q + ((b * G.n_tot + n) * G.Hd + h) * G.D;
    std::vector<double> s(keys.size());
    double m = -INFINITY;
    for (size_t c = 0; c < keys.size(); ++c) {
      const float* kv = k + ((b * G.n_tot + keys[c]) * G.Hd + h) * G.D;
      double acc = 0.0;
      for (long long d = 0; d < G.D; ++d) acc += (double)qv[d] * (double)kv[d];
      s[c] = acc * scale;
      m = std::max(m, s[c]);
    }
    double z = 0.0;
    for (size_t c = 0; c < keys.size(); ++c) {
      s[c] = std::exp(s[c] - m);
      z += s[c];
    }
    double* out = o + ((b * nr + r) * G.Hd + h) * G.D;
    for (long long d = 0; d < G.D; ++d) out[d] = 0.0;
    for (size_t c = 0; c < keys.size(); ++c) {
      const float* vv = v + ((b * G.n_tot + keys[c]) * G.Hd + h) * G.D;
      double w = s[c] / z;
      for (long long d = 0; d < G.D; ++d) out[d] += w * (double)vv[d];
    }
  });
}

// Box summarizer (SPADE §3.1 DSA-SPADE / DSA2-SPADE summaries k_max, k_min,
// q_max, q_min; §3.2 "The Summarizer Expression reduces over sequence
// positions of Q/K (e.g., max/min/mean)"): per video block and dimension the
// maximum and the minimum over the block's valid tokens.
// x [B, Ntot, Hd, D] -> box [B, Hd, nb, D, 2] with (max, min) pairs.
void orc_box_summaries(const int* g, const float* x, double* box) {
  Geom G = make_geom(g);
  parallel_for(G.B * G.Hd * G.nb, [&](long long task) {
    long long b = task / (G.Hd * G.nb), h = (task / G.nb) % G.Hd, j = task % G.nb;
    std::vector<long long> toks = block_tokens(G, j);
    double* out = box + task * G.D * 2;
    for (long long d = 0; d < G.D; ++d) {
      double mx = -INFINITY, mn = INFINITY;
      for (long long t : toks) {
        double v = (double)x[((b * G.n_tot + t) * G.Hd + h) * G.D + d];
        mx = std::max(mx, v);
        mn = std::min(mn, v);
      }
      out[2 * d] = mx;
      out[2 * d + 1] = mn;
    }
  });
}

// Inter-block scores from box summaries, then the row softmax (R4).
// variant 1, DSA-SPADE (estimate with (k_max, k_min, (q_max + q_min)/2)),
//   reading R21: the largest value of c . k over the key block's box,
//   c = (q_max + q_min) / 2, i.e. sum_d max(c_d k_max_d, c_d k_min_d);
// variant 2, DSA2-SPADE (estimate with (k_max, k_min, q_max, q_min)),
//   reading R21: the largest value of q . k over the query box times the key
//   box, i.e. sum_d max over the four corner products of dimension d;
// s_ij = estimate / sqrt(D), p_i = softmax_j(s_i).
void orc_scores_box(const int* g, const double* qbox, const double* kbox, int variant,
                    double* p) {
  Geom G = make_geom(g);
  const double scale = 1.0 / std::sqrt((double)G.D);
  parallel_for(G.B * G.Hd * G.nb, [&](long long row) {
    long long bh = row / G.nb;
    const double* qb = qbox + row * G.D * 2;
    double* pr = p + row * G.nb;
    for (long long j = 0; j < G.nb; ++j) {
      const double* kb = kbox + (bh * G.nb + j) * G.D * 2;
      double est = 0.0;
      for (long long d = 0; d < G.D; ++d) {
        const double qM = qb[2 * d], qm = qb[2 * d + 1], kM = kb[2 * d], km = kb[2 * d + 1];
        if (variant == 1) {
          const double c = (qM + qm) / 2.0;
          est += std::max(c * kM, c * km);
        } else {
          est += std::max(std::max(qM * kM, qM * km), std::max(qm * kM, qm * km));
        }
      }
      pr[j] = est * scale;
    }
    double mx = -INFINITY;
    for (long long j = 0; j < G.nb; ++j) mx = std::max(mx, pr[j]);
    double z = 0.0;
    for (long long j = 0; j < G.nb; ++j) {
      pr[j] = std::exp(pr[j] - mx);
      z += pr[j];
    }
    for (long long j = 0; j < G.nb; ++j) pr[j] /= z;
  });
}

// Intra-block estimator (SPADE §3.2, Eq. (4)): the sum over all ordered pairs
// (a, b) of valid tokens of a block of the cosine similarity
// q_a.q_b / (|q_a| |q_b|), diagonal included.  Reading R15: a zero vector has
// no direction and contributes nothing.  x [B, Ntot, Hd, D] -> out [B, Hd, nb].
void orc_sics(const int* g, const float* x, double* out) {
  Geom G = make_geom(g);
  parallel_for(G.B * G.Hd * G.nb, [&](long long task) {
    long long b = task / (G.Hd * G.nb), h = (task / G.nb) % G.Hd, j = task % G.nb;
    std::vector<long long> toks = block_tokens(G, j);
    std::vector<double> u(toks.size() * G.D, 0.0);
    for (size_t a = 0; a < toks.size(); ++a) {
      const float* v = x + ((b * G.n_tot + toks[a]) * G.Hd + h) * G.D;
      double nrm = 0.0;
      for (long long d = 0; d < G.D; ++d) nrm += (double)v[d] * (double)v[d];
      nrm = std::sqrt(nrm);
      if (nrm > 0.0)
        for (long long d = 0; d < G.D; ++d) u[a * G.D + d] = (double)v[d] / nrm;
    }
    double s = 0.0;
    for (size_t a = 0; a < toks.size(); ++a)
      for (size_t c = 0; c < toks.size(); ++c) {
        double dot = 0.0;
        for (long long d = 0; d < G.D; ++d) dot += u[a * G.D + d] * u[c * G.D + d];
        s += dot;
      }
    out[task] = s;
  });
}

// The same quantity by the online form of SPADE §3.2 (Eq. (5), Algorithm 1):
// walk the block's vectors in slot order, keeping the running sum r of the
// normalised vectors seen so far and sigma += <r, qhat_j> before adding
// qhat_j; the result is 2*sigma + (number of nonzero vectors).
void orc_sics_online(const int* g, const float* x, double* out) {
  Geom G = make_geom(g);
  parallel_for(G.B * G.Hd * G.nb, [&](long long task) {
    long long b = task / (G.Hd * G.nb), h = (task / G.nb) % G.Hd, j = task % G.nb;
    std::vector<long long> toks = block_tokens(G, j);
    std::vector<double> r(G.D, 0.0), qh(G.D);
    double sigma = 0.0;
    long long n = 0;
    for (long long t : toks) {
      const float* v = x + ((b * G.n_tot + t) * G.Hd + h) * G.D;
      double nrm = 0.0;
      for (long long d = 0; d < G.D; ++d) nrm += (double)v[d] * (double)v[d];
      nrm = std::sqrt(nrm);
      if (nrm == 0.0) continue;
      double dot = 0.0;
      for (long long d = 0; d < G.D; ++d) {
        qh[d] = (double)v[d] / nrm;
        dot += r[d] * qh[d];
      }
      sigma += dot;
      for (long long d = 0; d < G.D; ++d) r[d] += qh[d];
      ++n;
    }
    out[task] = 2.0 * sigma + (double)n;
  });
}

// Aggregation score (SPADE §3.2, Eq. (3)): AS = sum over the video blocks of
// SICS, per batch element and head.  as [B, Hd].
void orc_aggregation_score(const int* g, const float* x, double* as) {
  Geom G = make_geom(g);
  std::vector<double> sics(G.B * G.Hd * G.nb);
  orc_sics(g, x, sics.data());
  for (long long bh = 0; bh < G.B * G.Hd; ++bh) {
    double s = 0.0;
    for (long long j = 0; j < G.nb; ++j) s += sics[bh * G.nb + j];
    as[bh] = s;
  }
}

// Number of (query token, key token) pairs the lists select, valid tokens
// only, per batch element and head summed (SPADE §4.1 "Sparsity — fraction of
// pruned attention scores"; effective FLOPs = 4 * pairs * D).
long long orc_selected_pairs(const int* g, const int* idx, const int* cnt,
                             int kmax) {
  Geom G = make_geom(g);
  std::vector<long long> valid(G.nb + G.nb_text);
  for (long long j = 0; j < G.nb + G.nb_text; ++j)
    valid[j] = (long long)block_tokens(G, j).size();
  long long total = 0;
  for (long long bh = 0; bh < G.B * G.Hd; ++bh) {
    for (long long i = 0; i < G.nb; ++i) {
      long long keys = 0;
      const int* list = idx + (bh * G.nb + i) * kmax;
      for (int e = 0; e < cnt[bh * G.nb + i]; ++e) keys += valid[list[e]];
      total += keys * valid[i];
    }
    for (long long i = G.nb; i < G.nb + G.nb_text; ++i)
      total += valid[i] * G.n_tot;
  }
  return total;
}

}  // extern "C"
