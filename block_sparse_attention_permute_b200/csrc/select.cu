// select.cu — index search: centroid score matrix + head-wise Top-K / Top-P.
//
// SPADE (arXiv 2608.03335) §3.3: "From Q'/K' we compute ... an inter-block
// importance matrix of size N_Qblocks x N_Kblocks via the inter-estimator.
// Scores are filtered by Top-K or Top-P."  §3.1: MEAN-SPADE estimates with
// (q_mean, k_mean); "the dot product of blue vectors gives inter-block
// importance"; Top-K keep or Top-P cumulative threshold per head.
//
// Scores: s_ij = qbar_i . kbar_j * (1/sqrt(D)) in fp32 (one fma chain over d
// in ascending order, so the value does not depend on the launch shape);
// p_ij = e_ij / Z_i with e_ij = expf(s_ij - max_j s_ij) and Z_i summed in fp64.
// Selection, one warp per query-block row:
//   Top-K: the k-th largest score is found by a bitwise search (at most 32
//          steps) over the order-preserving integer image of s; equal scores
//          are taken in ascending block id.
//   Top-P: the largest score threshold whose mass sum_{s_j >= t} e_j reaches
//          tau * Z (fp64), then ties at the threshold in ascending block id
//          until the mass is reached: the shortest prefix in descending order.
// Lists are written in ascending block id; the text key blocks follow.
#include "kernels.cuh"

namespace bsa {


constexpr int kSelRows = 16;      // query-block rows per CTA (8 for long rows, see launch_select_t)
constexpr int kSelDChunk = 8;    // head-dim slice of a key chunk held in shared memory
constexpr int kSelBufs = 2;      // key-chunk buffers (2: the next chunk lands while one is used)
constexpr int kSelKS = kSelDChunk + 4;   // padded chunk row: conflict-free float4 reads
constexpr int kSelThreads = 256;  // 8 warps

// query summaries, the key-chunk buffers, the score rows
size_t select_smem_bytes(int nb, int D, int rows, int kpt) {
  return sizeof(float) * ((size_t)rows * D + kSelBufs * (size_t)(128 * kpt) * kSelKS + (size_t)rows * nb);
}

__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Sum over the warp, the same value in every lane (tree to lane 0, broadcast).
__device__ __forceinline__ double warp_sum_uniform(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  return __shfl_sync(0xffffffffu, v, 0);
}

__device__ __forceinline__ int warp_count(bool pred) {
  return __popc(__ballot_sync(0xffffffffu, pred));
}

// Weight of a score in the Top-P mass: expf(s - m) for the softmax of the
// inter-block scores, the score itself for intra scores.
struct SoftmaxWeight {
  float m;
  __device__ __forceinline__ double operator()(float s) const { return (double)expf(s - m); }
};
struct PlainWeight {
  __device__ __forceinline__ double operator()(float s) const { return (double)s; }
};

// sum over j with key(s_j) >= cand of wt(s_j), in fp64, fixed order.
template <class Wt>
__device__ double mass_at_least(const float* row, int nb, Wt wt, uint32_t cand, int lane) {
  double acc = 0.0;
  for (int j = lane; j < nb; j += 32) {
    const float s = row[j];
    if (order_key(s) >= cand) acc += wt(s);
  }
  return warp_sum_uniform(acc);
}

__device__ int count_at_least(const float* row, int nb, uint32_t cand, int lane) {
  int c = 0;
  for (int j = lane; j < nb; j += 32) c += order_key(row[j]) >= cand ? 1 : 0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
  return c;
}

// Lanes hold the order keys of their scores (j = lane + 32 e) in registers
// (and, for Top-P, their weights), so the 32-step threshold search neither
// re-reads shared memory nor recomputes a weight; the register count per
// lane is the smallest of 16, 32, 48 that covers the row.
constexpr int kKeysPerLane = 48;   // register-resident search for nb <= 1536

// Threshold of the Top-K / Top-P rule over one row with the keys (and, for
// Top-P, the weights) in registers.  Every sum runs over j = lane + 32 e in
// ascending e, then across the warp, as in mass_at_least, so the fp64 masses
// are those of the shared-memory loops below.
template <int KPL, bool TOPP, class Wt>
__device__ __forceinline__ void rule_threshold_regs(const float* row, int nb, int k, double target,
                                                    Wt wt, int lane, uint32_t* T_out, int* need_out) {
  // order_key of any float is nonzero and every candidate threshold is
  // nonzero, so the 0 used for missing entries never counts
  uint32_t kr[KPL];
  float wf[TOPP ? KPL : 1];   // weight of each score (0 for missing entries)
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = lane + 32 * e;
    const float sv = j < nb ? row[j] : 0.f;
    kr[e] = j < nb ? order_key(sv) : 0u;
    if (TOPP) wf[e] = j < nb ? (float)wt(sv) : 0.f;
  }
  uint32_t T = 0;
  int need = 0;
  if (!TOPP) {
    // Once exactly k keys reach a candidate, {key >= cand} is the Top-K set
    // (the same set the full search's threshold, the k-th key, selects) and
    // the search can stop there.
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int c = 0;
#pragma unroll
      for (int e = 0; e < KPL; ++e) c += kr[e] >= cand ? 1 : 0;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= k) {
        T = cand;
        if (c == k) break;
      }
    }
    int c = 0;
#pragma unroll
    for (int e = 0; e < KPL; ++e) c += kr[e] > T ? 1 : 0;
    need = k - __reduce_add_sync(0xffffffffu, c);
  } else {
    // mass of the keys >= cand; a weight is a float widened exactly to fp64
    auto mass = [&](uint32_t cand) -> double {
      double acc = 0.0;
#pragma unroll
      for (int e = 0; e < KPL; ++e)
        if (kr[e] >= cand) acc += (double)wf[TOPP ? e : 0];   // cand >= 1: missing entries never count
      return warp_sum_uniform(acc);
    };
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      if (mass(cand) >= target) T = cand;
    }
    double acc = (T == 0xffffffffu) ? 0.0 : mass(T + 1);
    int n_eq = 0;
    float s_eq = 0.f;
#pragma unroll
    for (int e = 0; e < KPL; ++e)
      if (kr[e] == T && lane + 32 * e < nb) { ++n_eq; s_eq = row[lane + 32 * e]; }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, off);
      s_eq = fmaxf(s_eq, __shfl_xor_sync(0xffffffffu, s_eq, off));
    }
    const double e_eq = wt(s_eq);
    while (acc < target && need < n_eq) {
      acc += e_eq;
      ++need;
    }
    if (need == 0) need = 1;
  }
  *T_out = T;
  *need_out = need;
}

// Threshold of the Top-K / Top-P rule over one row of nb scores: every entry
// with order key > T is taken, plus the first `need` (ascending j) of those
// with key == T.  Top-K: param = k.  Top-P: param = tau, `total` = the sum of
// all weights; the shortest descending prefix whose weight reaches
// tau * total (at least one entry).
// KMAX: the most keys per lane this instance keeps in registers (0: none,
// every row takes the shared-memory loops); the launch picks the smallest
// that covers its rows, so short rows do not pay for the registers of long
// ones.
template <int KMAX, class Wt>
__device__ __forceinline__ void rule_threshold(const float* row, int nb, int mode, double param,
                                               double total, Wt wt, int lane, uint32_t* T_out,
                                               int* need_out) {
  uint32_t T = 0;
  int need = 0;
  const double target = param * total;
  if (mode != 0 && !(target > 0.0)) {   // every prefix reaches 0: one entry
    mode = 0;
    param = 1.0;
  }
  // Registers: Top-K keeps up to 48 keys per lane, Top-P up to 32 keys and
  // their weights; longer rows use the shared-memory loops.
  if constexpr (KMAX >= 16) {
    if (mode == 0 && nb <= 32 * 16) {
      rule_threshold_regs<16, false>(row, nb, (int)param, target, wt, lane, T_out, need_out);
      return;
    }
    if (mode != 0 && nb <= 32 * 16) {
      rule_threshold_regs<16, true>(row, nb, 0, target, wt, lane, T_out, need_out);
      return;
    }
  }
  if constexpr (KMAX >= 32) {
    if (mode == 0 && nb <= 32 * 32) {
      rule_threshold_regs<32, false>(row, nb, (int)param, target, wt, lane, T_out, need_out);
      return;
    }
    if (mode != 0 && nb <= 32 * 32) {
      rule_threshold_regs<32, true>(row, nb, 0, target, wt, lane, T_out, need_out);
      return;
    }
  }
  if constexpr (KMAX >= kKeysPerLane) {
    if (mode == 0 && nb <= 32 * kKeysPerLane) {
      rule_threshold_regs<kKeysPerLane, false>(row, nb, (int)param, target, wt, lane, T_out, need_out);
      return;
    }
  }
  if (mode == 0) {
    const int k = (int)param;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      if (count_at_least(row, nb, cand, lane) >= k) T = cand;
    }
    const int n_gt = (T == 0xffffffffu) ? 0 : count_at_least(row, nb, T + 1, lane);
    need = k - n_gt;
  } else {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      if (mass_at_least(row, nb, wt, cand, lane) >= target) T = cand;
    }
    double acc = (T == 0xffffffffu) ? 0.0 : mass_at_least(row, nb, wt, T + 1, lane);
    int n_eq = 0;
    float s_eq = 0.f;
    for (int j = lane; j < nb; j += 32)
      if (order_key(row[j]) == T) { ++n_eq; s_eq = row[j]; }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, off);
      s_eq = fmaxf(s_eq, __shfl_xor_sync(0xffffffffu, s_eq, off));
    }
    const double e_eq = wt(s_eq);
    while (acc < target && need < n_eq) {
      acc += e_eq;
      ++need;
    }
    if (need == 0) need = 1;
  }
  *T_out = T;
  *need_out = need;
}

// First token (in the original order) of video block j: its corner.
__device__ __forceinline__ long long block_first_token(const Geo& g, int j) {
  const int xb = j % g.nbx, yb = (j / g.nbx) % g.nby, tb = j / (g.nbx * g.nby);
  return ((long long)tb * g.bf * g.H + (long long)yb * g.br) * g.W + (long long)xb * g.bc;
}

// Largest product of a in [am, aM] and b in [bm, bM] (a corner of the box).
__device__ __forceinline__ float box_max_product(float aM, float am, float bM, float bm) {
  return fmaxf(fmaxf(aM * bM, aM * bm), fmaxf(am * bM, am * bm));
}

// D = length of the stored summary vectors (head_dim for MEAN, 2 * head_dim
// for the (max, min) boxes of DSA and DSA2).
// KPT: keys per thread in a score chunk of 128 * KPT key blocks (2: chunks
// of 256; 3 where a row of nb keys pads less in chunks of 384, e.g. Wan's
// nb = 336: 48 idle key slots instead of 176, 15-17 % less selection time).
template <int D, int EST, int ROWS, int KMAX, int KPT>
__global__ void __launch_bounds__(kSelThreads, KMAX == 16 ? 3 : 2)
    select_kernel(Geo g, SelectArgs a) {
  constexpr int RPT = ROWS / 2;                     // rows per thread in phase 1
  constexpr int KC = 128 * KPT;                     // key blocks per score chunk
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                                   // [ROWS][D]
  float* ks = qs + ROWS * D;                        // [kSelBufs][KC][kSelKS]
  float* sc = ks + kSelBufs * KC * kSelKS;          // [ROWS][nb]
  const int nb = g.nb;
  const int bhi = map_bh(a.map, (int)blockIdx.z * g.Hd + (int)blockIdx.y);
  const int h = bhi % g.Hd, b = bhi / g.Hd;
  const long long bh = (long long)b * g.Hd + h;
  const int i0 = blockIdx.x * ROWS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- phase 1: scores of ROWS query blocks against all key blocks ----
  // Thread (ty, tx) accumulates rows RPT ty .. RPT ty + RPT - 1 against keys tx + 128 k
  // (k < KPT) of each KC-key chunk; the chunk's keys pass through shared memory 8
  // dimensions at a time (double-buffered).  Each dot product is one fma chain over d in
  // ascending order, the same as a plain sequential loop.
  if (EST == kEstDsa) {
    // DSA: the query summary is the box centre c = (max + min) / 2, stored as
    // (c+, c-) pairs so that c+ kmax + c- kmin = max(c kmax, c kmin)
    for (int e = tid; e < ROWS * D / 2; e += kSelThreads) {
      const int r = e / (D / 2), d = e % (D / 2);
      float cp = 0.f, cn = 0.f;
      if (i0 + r < nb) {
        const float* src = a.qc + (bh * nb + i0 + r) * D + 2 * d;
        const float c = 0.5f * (src[0] + src[1]);
        cp = fmaxf(c, 0.f);
        cn = fminf(c, 0.f);
      }
      qs[r * D + 2 * d] = cp;
      qs[r * D + 2 * d + 1] = cn;
    }
  } else {
    for (int e = tid; e < ROWS * D; e += kSelThreads) {
      const int r = e / D, d = e % D;
      qs[e] = (i0 + r < nb) ? a.qc[(bh * nb + i0 + r) * D + d] : 0.f;
    }
  }
  const int ty = tid / 128, tx = tid % 128;
  // The key chunks (KC key blocks x kSelDChunk dimensions) are visited
  // j0-major; chunk c + 1 is copied with cp.async into the other buffer while
  // chunk c is used.  Rows past nb are zero-filled.
  constexpr int kDChunks = D / kSelDChunk;
  const int n_chunks = ((nb + KC - 1) / KC) * kDChunks;
  const float* kc_bh = a.kc + bh * nb * D;
  auto issue_chunk = [&](int c) {
    const int j0 = (c / kDChunks) * KC, d0 = (c % kDChunks) * kSelDChunk;
    float* buf = ks + (c % kSelBufs) * KC * kSelKS;
    for (int e = tid; e < KC * (kSelDChunk / 4); e += kSelThreads) {
      const int jj = e / (kSelDChunk / 4), d4 = e % (kSelDChunk / 4);
      const bool ok = j0 + jj < nb;
      cp_async16(smem_addr(buf + jj * kSelKS + 4 * d4),
                 ok ? kc_bh + (long long)(j0 + jj) * D + d0 + 4 * d4 : kc_bh, ok ? 16u : 0u);
    }
    cp_async_commit();
  };
  if (kSelBufs == 2) issue_chunk(0);
  float acc[RPT][KPT];
  for (int c = 0; c < n_chunks; ++c) {
    const int j0 = (c / kDChunks) * KC, d0 = (c % kDChunks) * kSelDChunk;
    if (d0 == 0) {
#pragma unroll
      for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int kp = 0; kp < KPT; ++kp) acc[r][kp] = 0.f;
    }
    if (kSelBufs == 1) {
      issue_chunk(c);
      cp_async_wait<0>();
    } else if (c + 1 < n_chunks) {
      issue_chunk(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();   // chunk c (and, at c = 0, the query summaries) visible
    const float* kb = ks + (c % kSelBufs) * KC * kSelKS;
#pragma unroll
    for (int d4 = 0; d4 < kSelDChunk / 4; ++d4) {
      float4 kv[KPT];
#pragma unroll
      for (int kp = 0; kp < KPT; ++kp)
        kv[kp] = *reinterpret_cast<const float4*>(kb + (tx + 128 * kp) * kSelKS + 4 * d4);
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (RPT * ty + r) * D + d0 + 4 * d4);
#pragma unroll
        for (int kp = 0; kp < KPT; ++kp) {
          if (EST == kEstDsa2) {
            acc[r][kp] += box_max_product(qv.x, qv.y, kv[kp].x, kv[kp].y);
            acc[r][kp] += box_max_product(qv.z, qv.w, kv[kp].z, kv[kp].w);
            continue;
          }
          acc[r][kp] = fmaf(qv.x, kv[kp].x, acc[r][kp]);
          acc[r][kp] = fmaf(qv.y, kv[kp].y, acc[r][kp]);
          acc[r][kp] = fmaf(qv.z, kv[kp].z, acc[r][kp]);
          acc[r][kp] = fmaf(qv.w, kv[kp].w, acc[r][kp]);
        }
      }
    }
    if (d0 + kSelDChunk == D) {
#pragma unroll
      for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int kp = 0; kp < KPT; ++kp)
          if (j0 + tx + 128 * kp < nb)
            sc[(RPT * ty + r) * nb + j0 + tx + 128 * kp] = acc[r][kp] * a.scale + 0.0f;
    }
    __syncthreads();   // buffer (c & 1) is refilled by the copy issued next iteration
  }
  __syncthreads();

  // ---- phase 2: one warp per row: softmax statistics and selection ----
  for (int r = warp; r < ROWS; r += kSelThreads / 32) {
    const int i = i0 + r;
    if (i >= nb) break;
    const float* row = sc + r * nb;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    // The normaliser is needed only for the score output and for Top-P
    // (Top-K depends on the order of the scores alone).
    const double Z = (a.scores != nullptr || a.mode != 0)
                         ? mass_at_least(row, nb, SoftmaxWeight{m}, 0u, lane) : 1.0;

    if (a.scores != nullptr) {
      float* out = a.scores + (bh * nb + i) * nb;
      for (int j = lane; j < nb; j += 32) out[j] = (float)((double)expf(row[j] - m) / Z);
    }

    uint32_t T = 0;
    int need = 0;  // how many of the scores equal to the threshold to take
    rule_threshold<KMAX>(row, nb, a.mode, a.param[h], Z, SoftmaxWeight{m}, lane, &T, &need);

    // Ascending compaction of {key > T} plus the first `need` of {key == T},
    // united with the window, sink and intra blocks.
    int32_t* out = a.idx + (bh * nb + i) * a.kmax;
    int written = 0, eq_seen = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const bool window = a.win_left >= 0 || a.win_right >= 0;
    const long long w_lo = a.win_left < 0 ? 0 : (long long)i - a.win_left;
    const long long w_hi = a.win_right < 0 ? nb : (long long)i + a.win_right;
    const int nbw = (nb + 31) / 32;
    const uint32_t* ibits = a.intra_bits ? a.intra_bits + bh * nbw : nullptr;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < nb ? order_key(row[j]) : 0u;
      const bool gt = j < nb && key > T;
      const bool eq = j < nb && key == T;
      const uint32_t eq_bal = __ballot_sync(0xffffffffu, eq);
      bool take = gt || (eq && eq_seen + __popc(eq_bal & lt_mask) < need);
      if (j < nb) {
        take = take || (window && j >= w_lo && j <= w_hi);
        take = take || (a.sink_tokens > 0 && block_first_token(g, j) < a.sink_tokens);
        take = take || (ibits != nullptr && ((ibits[j >> 5] >> (j & 31)) & 1u));
      }
      const uint32_t sel_bal = __ballot_sync(0xffffffffu, take);
      if (take) out[written + __popc(sel_bal & lt_mask)] = j;
      if (a.list_bits != nullptr && lane == 0) a.list_bits[(bh * nb + i) * nbw + (j0 >> 5)] = sel_bal;
      written += __popc(sel_bal);
      eq_seen += __popc(eq_bal);
    }
    for (int t = lane; t < g.nb_text; t += 32) out[written + t] = nb + t;
    if (lane == 0) a.cnt[bh * nb + i] = written + g.nb_text;
  }
}

// Intra selection (SPADE §3.3: intra scores, one per block, filtered by the
// intra-top value and broadcast to every query block): per (b, h) the same
// Top-K / Top-P rule on the intra scores, with a score's own value as its
// Top-P weight; the selected key blocks are written as a bit set.
constexpr int kIntraWarps = 4;

__global__ void __launch_bounds__(kIntraWarps * 32) intra_select_kernel(Geo g, IntraArgs a) {
  const int slot = blockIdx.x * kIntraWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (slot >= map_count(a.map, g.B * g.Hd)) return;
  const int bh = map_bh(a.map, slot);
  const int nb = g.nb, nbw = (nb + 31) / 32, h = bh % g.Hd;
  const float* row = a.scores + (long long)bh * nb;
  uint32_t* bits = a.bits + (long long)bh * nbw;
  const double prm = a.param[h];
  if (!(prm > 0.0)) {
    for (int w = lane; w < nbw; w += 32) bits[w] = 0u;
    return;
  }
  const double total = a.mode != 0 ? mass_at_least(row, nb, PlainWeight{}, 0u, lane) : 0.0;
  uint32_t T = 0;
  int need = 0;
  rule_threshold<kKeysPerLane>(row, nb, a.mode, prm, total, PlainWeight{}, lane, &T, &need);
  int eq_seen = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < nb ? order_key(row[j]) : 0u;
    const bool gt = j < nb && key > T;
    const bool eq = j < nb && key == T;
    const uint32_t eq_bal = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eq_bal & lt_mask) < need);
    const uint32_t sel_bal = __ballot_sync(0xffffffffu, take);
    if (lane == 0) bits[j0 >> 5] = sel_bal;
    eq_seen += __popc(eq_bal);
  }
}

cudaError_t launch_intra_select(const Geo& g, const IntraArgs& a, cudaStream_t st) {
  const int BH = map_count(a.map, g.B * g.Hd);
  if (BH == 0 || g.nb == 0) return cudaSuccess;
  intra_select_kernel<<<(BH + kIntraWarps - 1) / kIntraWarps, kIntraWarps * 32, 0, st>>>(g, a);
  return cudaGetLastError();
}

template <int D, int EST, int ROWS, int KMAX, int KPT = 2>
static cudaError_t launch_select_rows(const Geo& g, const SelectArgs& a, cudaStream_t st) {
  const size_t smem = select_smem_bytes(g.nb, D, ROWS, KPT);
  // with a head map, y enumerates its pairs (z = 1) and the kernel reads
  // map_bh(y); without one, y = h and z = b
  dim3 grid((g.nb + ROWS - 1) / ROWS, a.map.n ? a.map.n : g.Hd, a.map.n ? 1 : g.B);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D, EST, ROWS, KMAX, KPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<D, EST, ROWS, KMAX, KPT><<<grid, kSelThreads, smem, st>>>(g, a);
  return cudaGetLastError();
}

// Rows of up to 512 / 1024 / 1536 key blocks keep 16 / 32 / 48 keys per lane
// in registers (16 keys fit in 80 registers: three CTAs per SM), longer rows
// none.  16 query rows per CTA while two CTAs fit on an SM; long rows (their
// scores fill shared memory) take 8 rows per CTA so that two CTAs still fit.
template <int D, int EST>
static cudaError_t launch_select_t(const Geo& g, const SelectArgs& a, cudaStream_t st) {
  constexpr size_t kTwoPerSm = 112 * 1024;
  const bool rows16 = select_smem_bytes(g.nb, D, kSelRows) <= kTwoPerSm;
  // rows in (256, 384] (Wan's 336 blocks) waste less in one chunk of 384 keys
  const bool kpt3 = g.nb > 256 && g.nb <= 384 && select_smem_bytes(g.nb, D, kSelRows, 3) <= kTwoPerSm;
  if (g.nb <= 32 * 16 && kpt3) return launch_select_rows<D, EST, kSelRows, 16, 3>(g, a, st);
  if (g.nb <= 32 * 16 && rows16) return launch_select_rows<D, EST, kSelRows, 16>(g, a, st);
  if (g.nb <= 32 * 32 && rows16) return launch_select_rows<D, EST, kSelRows, 32>(g, a, st);
  if (g.nb <= 32 * kKeysPerLane)
    return rows16 ? launch_select_rows<D, EST, kSelRows, kKeysPerLane>(g, a, st)
                  : launch_select_rows<D, EST, 8, kKeysPerLane>(g, a, st);
  return rows16 ? launch_select_rows<D, EST, kSelRows, 0>(g, a, st)
                : launch_select_rows<D, EST, 8, 0>(g, a, st);
}

cudaError_t launch_select(const Geo& g, const SelectArgs& a, cudaStream_t st) {
  const bool d128 = g.D == 128;
  switch (a.est) {
    case kEstDsa:
      return d128 ? launch_select_t<256, kEstDsa>(g, a, st) : launch_select_t<128, kEstDsa>(g, a, st);
    case kEstDsa2:
      return d128 ? launch_select_t<256, kEstDsa2>(g, a, st) : launch_select_t<128, kEstDsa2>(g, a, st);
    default:
      return d128 ? launch_select_t<128, kEstMean>(g, a, st) : launch_select_t<64, kEstMean>(g, a, st);
  }
}

}  // namespace bsa
