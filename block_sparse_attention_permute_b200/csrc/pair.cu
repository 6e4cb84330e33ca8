// pair.cu — pairing of the query tiles of each (batch, head) for the
// attention kernel, so that the two tiles of a CTA share key blocks.
//
// The attention kernel runs two query tiles per CTA.  Block-sparse lists
// differ per query block, so two arbitrary tiles rarely need the same K/V
// tiles; but the lists of query blocks with similar summaries overlap
// strongly.  Here each (b, h)'s video query blocks are matched in pairs with
// large overlap |L_i & L_j|: every block keeps its kCand best partners among
// its neighbours in block order (a window reaching the next frame), and
// in a few "mutual best partner" rounds a block and its best unmatched
// candidate are matched when each is the other's; the rest are paired in
// index order.  Each pair's two lists are reordered so that the shared
// blocks come first, in the same order, followed by the text blocks (shared
// by every list) and then each tile's own blocks.  For those first c steps
// the attention kernel fetches every K and V tile once for both tiles.  The
// order of a list's blocks is free (softmax is order independent; only the
// rounding of the sums moves).
#include "kernels.cuh"

namespace bsa {

constexpr int kPairRounds = 4;
constexpr int kMaxWords = 48;   // nb <= 1536
constexpr int kCand = 8;        // candidate partners kept per query block

bool pairing_supported(const Geo& g) { return g.nb <= 32 * kMaxWords; }

size_t pair_scratch_bytes(const Geo& g) {
  const size_t nbw = (g.nb + 31) / 32;
  const size_t bh = (size_t)g.B * g.Hd;
  return bh * g.nb * nbw * sizeof(uint32_t) + 256 + bh * g.nb * kCand * sizeof(uint16_t);
}

// Bit set of the video blocks of every list: one warp per (bh, i), the list
// read 32 entries at a time and the bits set with shared-memory atomics.
__global__ void __launch_bounds__(256) pair_bits_kernel(Geo g, PairArgs a) {
  __shared__ uint32_t s_bits[8][kMaxWords];
  const int bh = map_bh(a.map, blockIdx.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * 8 + warp;
  if (i >= g.nb) return;
  const int nbw = (g.nb + 31) / 32;
  for (int w = lane; w < kMaxWords; w += 32) s_bits[warp][w] = 0u;
  __syncwarp();
  const int32_t* L = a.idx + ((long long)bh * g.nb + i) * a.kmax;
  int n = a.cnt[(long long)bh * g.nb + i];
  n = n < 0 ? 0 : (n > a.kmax ? a.kmax : n);
  for (int s = lane; s < n; s += 32) {
    const int j = __ldg(L + s);
    if (j >= 0 && j < g.nb) atomicOr(&s_bits[warp][j >> 5], 1u << (j & 31));
  }
  __syncwarp();
  uint32_t* out = a.bits + ((long long)bh * g.nb + i) * nbw;
  for (int w = lane; w < nbw; w += 32) out[w] = s_bits[warp][w];
}

// Candidate partners of every query block: its kCand largest overlaps
// |L_i & L_j| over the blocks j within `win` of i in block order (j != i;
// equal overlaps to the smaller j).  The window covers the neighbours of a
// block in x, y and t (a t-neighbour is nbx * nby blocks away); blocks that
// far apart rarely share more keys than the near ones, and searching all nb
// blocks cost nb^2 popcount rows per head.  One warp per (bh, i), kCandRows
// rows per CTA; lane l holds the overlaps with j = i - win + l + 32 t in
// registers.  The bit sets of rows [i0 - win, i0 + kCandRows + win) are
// staged in shared memory with an odd row stride (conflict-free column reads).
constexpr int kCandRows = 16;
constexpr int kWinT = 8;   // at most 8 * 32 candidates per block: win <= 127

int pair_window_lanes(const Geo& g) {
  const long long w0 = (long long)g.nbx * g.nby + g.nbx + 1;
  const long long t = (2 * w0 + 1 + 31) / 32;
  return (int)(t < kWinT ? t : kWinT);
}
size_t pair_cand_smem(const Geo& g) {
  const int win = (32 * pair_window_lanes(g) - 1) / 2;
  const int nbw = (g.nb + 31) / 32;
  return (size_t)(kCandRows + 2 * win) * (nbw | 1) * sizeof(uint32_t);
}

__global__ void __launch_bounds__(kCandRows * 32) pair_cand_kernel(Geo g, PairArgs a, int n_t) {
  extern __shared__ uint32_t s_bits_all[];
  const int bh = map_bh(a.map, blockIdx.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = g.nb, nbw = (nb + 31) / 32, stride = nbw | 1;
  const int win = (32 * n_t - 1) / 2;
  const int i0 = blockIdx.y * kCandRows;
  const int lo = max(0, i0 - win), hi = min(nb, i0 + kCandRows + win);
  const uint32_t* gbits = a.bits + (long long)bh * nb * nbw;
  for (int e = threadIdx.x; e < (hi - lo) * nbw; e += blockDim.x)
    s_bits_all[(e / nbw) * stride + e % nbw] = gbits[(long long)lo * nbw + e];
  __syncthreads();
  const int i = i0 + warp;
  if (i >= nb) return;
  const uint32_t* row_i = s_bits_all + (i - lo) * stride;
  const int jbase = i - win;   // j of (lane 0, t = 0)
  int ov[kWinT];   // -1: no such j, or already picked
#pragma unroll
  for (int t = 0; t < kWinT; ++t) {
    const int j = jbase + lane + 32 * t;
    int c = -1;
    if (t < n_t && lane + 32 * t <= 2 * win && j >= 0 && j < nb && j != i) {
      c = 0;
      const uint32_t* row_j = s_bits_all + (j - lo) * stride;
      for (int w = 0; w < nbw; ++w) c += __popc(row_i[w] & row_j[w]);
    }
    ov[t] = c;
  }
  uint16_t* out = a.cand + ((long long)bh * nb + i) * kCand;
  for (int k = 0; k < kCand; ++k) {
    int bv = -1, bt = -1;
#pragma unroll
    for (int t = 0; t < kWinT; ++t)
      if (ov[t] > bv) { bv = ov[t]; bt = t; }
    int bj = bt >= 0 ? jbase + lane + 32 * bt : -1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const int v2 = __shfl_xor_sync(0xffffffffu, bv, o);
      const int j2 = __shfl_xor_sync(0xffffffffu, bj, o);
      if (v2 > bv || (v2 == bv && j2 >= 0 && (bj < 0 || j2 < bj))) { bv = v2; bj = j2; }
    }
    if (lane == 0) out[k] = bj < 0 ? (uint16_t)0xffffu : (uint16_t)bj;
    if (bj >= 0 && ((bj - jbase) & 31) == lane) {   // remove the pick from its lane
      const int tp = (bj - jbase) >> 5;
#pragma unroll
      for (int t = 0; t < kWinT; ++t)
        if (t == tp) ov[t] = -1;
    }
  }
}

// Exclusive prefix sum of one value per thread over the block (at most 1024
// threads); returns this thread's offset and sets *total.
__device__ __forceinline__ int block_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    s_warp[lane] = wi - w;
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  const int off = s_warp[warp] + incl - v;
  *total = s_warp[32];
  __syncthreads();
  return off;
}

// Writes, in ascending order from out[base], the block ids of the set bits
// of A & B (both), A & ~B (andnot) or A; the lanes share the words.
// Returns the number written.
__device__ __forceinline__ int write_bits(const uint32_t* wordsA, const uint32_t* wordsB, bool andnot,
                                          bool both, int nbw, int32_t* out, int base, int lane) {
  int written = 0;
  for (int w0 = 0; w0 < nbw; w0 += 32) {
    const int w = w0 + lane;
    uint32_t v = 0u;
    if (w < nbw) v = both ? (wordsA[w] & wordsB[w]) : (andnot ? (wordsA[w] & ~wordsB[w]) : wordsA[w]);
    const int c = __popc(v);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = base + written + incl - c;
    while (v) {
      const int b = __ffs(v) - 1;
      out[pos++] = w * 32 + b;
      v &= v - 1;
    }
    written += __shfl_sync(0xffffffffu, incl, 31);
  }
  return written;
}

// Matching of one (b, h): one CTA of 1024 threads, in shared memory; writes
// the tiles of every schedule entry.
__global__ void __launch_bounds__(1024) pair_match_kernel(Geo g, PairArgs a) {
  extern __shared__ int sm_pair[];
  const int nb = g.nb;
  int* partner = sm_pair;          // [nb] matched block, -1 = none
  int* best = partner + nb;        // [nb] best unmatched candidate this round
  int* pair_i = best + nb;         // [nb] first tile of pair p
  int* pair_j = pair_i + nb;       // [nb] second tile of pair p (-1: single)
  int* rest = pair_j + nb;         // [nb] unmatched blocks in index order
  __shared__ int s_scan[33];
  const int bh = map_bh(a.map, blockIdx.x);
  const uint16_t* cand = a.cand + (long long)bh * nb * kCand;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) partner[i] = -1;
  __syncthreads();
  for (int round = 0; round < kPairRounds; ++round) {
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
      int b = -1;
      if (partner[i] < 0) {
        for (int k = 0; k < kCand; ++k) {
          const int j = cand[(long long)i * kCand + k];
          if (j < nb && partner[j] < 0) { b = j; break; }
        }
      }
      best[i] = b;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
      const int j = best[i];
      if (partner[i] < 0 && j > i && partner[j] < 0 && best[j] == i) {
        partner[i] = j;
        partner[j] = i;
      }
    }
    __syncthreads();
  }
  // the unmatched blocks, in index order, are paired two by two
  int n_rest = 0;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int f = (i < nb && partner[i] < 0) ? 1 : 0;
    int tot;
    const int off = block_scan(f, s_scan, &tot);
    if (f) rest[n_rest + off] = i;
    n_rest += tot;
  }
  __syncthreads();
  for (int m = threadIdx.x; 2 * m + 1 < n_rest; m += blockDim.x) {
    partner[rest[2 * m]] = rest[2 * m + 1];
    partner[rest[2 * m + 1]] = rest[2 * m];
  }
  __syncthreads();
  // pairs in order of their first block (a lone block is a pair of one)
  int np = 0;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int f = (i < nb && (partner[i] < 0 || partner[i] > i)) ? 1 : 0;
    int tot;
    const int off = block_scan(f, s_scan, &tot);
    if (f) {
      pair_i[np + off] = i;
      pair_j[np + off] = partner[i];
    }
    np += tot;
  }
  __syncthreads();
  int32_t* sched = a.sched + (long long)bh * a.pairs_per_head * 4;
  // text pairs: dense rows, every step shared
  for (int t = threadIdx.x; t < a.text_pairs; t += blockDim.x) {
    const int i0 = nb + 2 * t, i1 = (2 * t + 1 < g.nb_text) ? nb + 2 * t + 1 : -1;
    sched[t * 4 + 0] = i0;
    sched[t * 4 + 1] = i1;
    sched[t * 4 + 2] = i1 >= 0 ? nb + g.nb_text : 0;
    sched[t * 4 + 3] = 0;
  }
  // video pairs: the tiles here, the shared count with the lists (next kernel)
  for (int p = threadIdx.x; p < a.pairs_per_head - a.text_pairs; p += blockDim.x) {
    const int e = a.text_pairs + p;
    sched[e * 4 + 0] = p < np ? pair_i[p] : -1;
    sched[e * 4 + 1] = p < np ? pair_j[p] : -1;
    sched[e * 4 + 2] = 0;
    sched[e * 4 + 3] = 0;
  }
}

// Reordered lists of every video pair (one warp per pair): the shared video
// blocks, the text blocks, then each tile's own blocks, all ascending; the
// shared count c goes into the schedule entry.
__global__ void __launch_bounds__(256) pair_lists_kernel(Geo g, PairArgs a) {
  const int vp = a.pairs_per_head - a.text_pairs;
  const int p = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (p >= vp) return;
  const int bh = map_bh(a.map, blockIdx.x);
  const int nb = g.nb, nbw = (nb + 31) / 32;
  const int e = a.text_pairs + p;
  int32_t* ent = a.sched + ((long long)bh * a.pairs_per_head + e) * 4;
  const int i = ent[0], j = ent[1];
  if (i < 0) return;
  const uint32_t* bits = a.bits + (long long)bh * nb * nbw;
  const uint32_t* bi = bits + (long long)i * nbw;
  int32_t* lists = a.lists + ((long long)bh * a.pairs_per_head + e) * 2 * a.kmax;
  int32_t* li = lists;
  int32_t* lj = lists + a.kmax;
  int c = 0;
  if (j >= 0) {
    const uint32_t* bj = bits + (long long)j * nbw;
    const int ns = write_bits(bi, bj, false, true, nbw, li, 0, lane);
    write_bits(bi, bj, false, true, nbw, lj, 0, lane);
    for (int t = lane; t < g.nb_text; t += 32) { li[ns + t] = nb + t; lj[ns + t] = nb + t; }
    c = ns + g.nb_text;
    write_bits(bi, bj, true, false, nbw, li, c, lane);
    write_bits(bj, bi, true, false, nbw, lj, c, lane);
  } else {
    const int ns = write_bits(bi, bi, false, false, nbw, li, 0, lane);
    for (int t = lane; t < g.nb_text; t += 32) li[ns + t] = nb + t;
  }
  if (lane == 0) ent[2] = c;
}

cudaError_t launch_pairing(const Geo& g, const PairArgs& a, cudaStream_t st) {
  const int n_bh = map_count(a.map, g.B * g.Hd);
  if (n_bh == 0 || g.nb == 0) return cudaSuccess;
  if (g.nb > 32 * kMaxWords) return cudaErrorInvalidValue;
  cudaError_t e;
  if (!a.bits_ready) {   // else the selection wrote the bit sets with the lists
    pair_bits_kernel<<<dim3(n_bh, (g.nb + 7) / 8), 256, 0, st>>>(g, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t cand_smem = pair_cand_smem(g);   // <= 270 rows x 49 words
  const dim3 cgrid(n_bh, (g.nb + kCandRows - 1) / kCandRows);
  e = cudaFuncSetAttribute(pair_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cand_smem);
  if (e != cudaSuccess) return e;
  pair_cand_kernel<<<cgrid, kCandRows * 32, cand_smem, st>>>(g, a, pair_window_lanes(g));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem = 5 * (size_t)g.nb * sizeof(int);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(pair_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  pair_match_kernel<<<n_bh, 1024, smem, st>>>(g, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int vp = a.pairs_per_head - a.text_pairs;
  pair_lists_kernel<<<dim3(n_bh, (vp + 7) / 8), 256, 0, st>>>(g, a);
  return cudaGetLastError();
}

}  // namespace bsa
