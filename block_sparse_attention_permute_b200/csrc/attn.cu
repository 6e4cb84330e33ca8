// attn.cu — flash block-sparse attention forward.
//
// SPADE (arXiv 2608.03335) §2.2 Eq. (2): softmax(QK^T/sqrt(d_k) + M) V with
// M = 0 on selected (query block, key block) pairs and valid keys, -inf
// elsewhere; §3.3 (3): "(i) preprocesses the mask into ranked BSR for
// sequential access, (ii) uses an online softmax to avoid materializing dense
// attention, and (iii) exploits [TMA and MMA units] to pipeline
// memory/compute".  The per-query-block index lists are the sparse rows.
//
// Two kernels:
//  * attn_tc_kernel (bf16, 128-token blocks, D in {64,128}): one CTA per two
//    query tiles (a pair of the tile-pairing schedule, or two consecutive
//    tiles); warp 8 issues TMA loads of the two Q tiles once and of the K/V
//    tiles of the selected key blocks only, through a 4-slot ring; warp 9
//    issues tcgen05.mma: S = Q K^T into TMEM, O += P V into TMEM, P read
//    from TMEM; warps 0-3 and 4-7 own one query row per thread of tile 0 and
//    tile 1: they read S from TMEM, apply the pad mask and the online softmax
//    (exp2 of log2e-prescaled logits, fp32 statistics, lazy rescaling of O in
//    TMEM), and write P (bf16) back into TMEM for the PV product.  The
//    epilogue divides by the row sum.  Details at the kernel.
//  * attn_simt_kernel (any dtype, any block size <= 256): one warp per query
//    row, fp32 scores and online softmax, exact fp32 arithmetic.  It serves
//    fp32 inputs and block shapes the tensor-core path does not take.
// Text query blocks (ids >= nb) attend every key block.
#include "kernels.cuh"

namespace bsa {


// Tile order: text query tiles first (they have the longest lists), then the
// video tiles, head-major so that one head's K/V stays resident in L2.
// The (batch, head) pairs come from the launch's head map (all of them when
// it is empty).
__device__ __forceinline__ void decode_tile(const Geo& g, const HeadMap& m, int L, int& b, int& h,
                                            int& i) {
  const int n_text_tiles = map_count(m, g.B * g.Hd) * g.nb_text;
  int slot;
  if (L < n_text_tiles) {
    i = g.nb + L % g.nb_text;
    slot = L / g.nb_text;
  } else {
    L -= n_text_tiles;
    i = L % g.nb;
    slot = L / g.nb;
  }
  const int bh = map_bh(m, slot);
  h = bh % g.Hd;
  b = bh / g.Hd;
}

__device__ __forceinline__ void set_status(int32_t* st, int code) {
  if (st != nullptr) atomicCAS(st, 0, code);
}

// List length of query block i (text rows are dense), clamped to [0, kmax].
__device__ __forceinline__ int list_length(const Geo& g, const AttnArgs& a, long long bh, int i) {
  if (i >= g.nb) return g.nb + g.nb_text;
  int n = __ldg(a.cnt + bh * g.nb + i);
  if (n < 0 || n > a.kmax) {
    set_status(a.status, 6);
    n = n < 0 ? 0 : a.kmax;
  }
  return n;
}

// ===========================================================================
// fp32 SIMT path
// ===========================================================================
template <typename T>
__device__ __forceinline__ float ld_elem(const T* p) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  else return *reinterpret_cast<const float*>(p);
}
template <typename T>
__device__ __forceinline__ void st_elem(T* p, float v) {
  if constexpr (sizeof(T) == 2) *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
  else *reinterpret_cast<float*>(p) = v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  return __shfl_sync(0xffffffffu, v, 0);
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

constexpr int kSimtWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kSimtWarps * 32) attn_simt_kernel(Geo g, AttnArgs a) {
  constexpr int DL = D / 32;  // elements of a row per lane
  __shared__ float s_q[kSimtWarps][D];
  int b, h, i;
  decode_tile(g, a.map, blockIdx.x, b, h, i);
  const long long bh = (long long)b * g.Hd + h;
  const int nbk = g.nb + g.nb_text;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Q = reinterpret_cast<const T*>(a.q);
  const T* K = reinterpret_cast<const T*>(a.k);
  const T* V = reinterpret_cast<const T*>(a.v);
  T* O = reinterpret_cast<T*>(a.o);
  const int n = list_length(g, a, bh, i);
  const int32_t* list = a.idx + (bh * g.nb + (i < g.nb ? i : 0)) * a.kmax;

  for (int r = warp; r < g.bs; r += kSimtWarps) {
    const long long qrow = (bh * nbk + i) * g.bs + r;
    T* orow = O + qrow * D;
    if (slot_token(g, i, r) < 0 || n == 0) {
      for (int d = lane; d < D; d += 32) st_elem(orow + d, 0.f);
      continue;
    }
    __syncwarp();
    for (int d = lane; d < D; d += 32) s_q[warp][d] = ld_elem(Q + qrow * D + d);
    __syncwarp();
    float m = -INFINITY, l = 0.f, acc[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[e] = 0.f;
    for (int s = 0; s < n; ++s) {
      const int j = i >= g.nb ? s : __ldg(list + s);
      if (j < 0 || j >= nbk) {
        set_status(a.status, 6);
        continue;
      }
      const long long krow0 = (bh * nbk + j) * g.bs;
      for (int c0 = 0; c0 < g.bs; c0 += 32) {
        const int c = c0 + lane;
        float sc = -INFINITY;
        if (c < g.bs && slot_token(g, j, c) >= 0) {
          const T* kr = K + (krow0 + c) * D;
          float dot = 0.f;
          for (int d = 0; d < D; ++d) dot = fmaf(s_q[warp][d], ld_elem(kr + d), dot);
          sc = dot * a.scale;
        }
        const float cmax = warp_max_f(sc);
        if (cmax == -INFINITY) continue;
        const float m_new = fmaxf(m, cmax);
        const float alpha = expf(m - m_new);
        const float p = (sc == -INFINITY) ? 0.f : expf(sc - m_new);
        l = l * alpha + warp_sum_f(p);
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] *= alpha;
        const int cn = min(32, g.bs - c0);
        for (int cc = 0; cc < cn; ++cc) {
          const float pc = __shfl_sync(0xffffffffu, p, cc);
          if (pc == 0.f) continue;
          const T* vr = V + (krow0 + c0 + cc) * D;
#pragma unroll
          for (int e = 0; e < DL; ++e) acc[e] = fmaf(pc, ld_elem(vr + lane + 32 * e), acc[e]);
        }
        m = m_new;
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) st_elem(orow + lane + 32 * e, acc[e] * inv);
  }
}

cudaError_t launch_attn_simt(const Geo& g, bool is_bf16, const AttnArgs& a, cudaStream_t st) {
  const int tiles = map_count(a.map, g.B * g.Hd) * (g.nb + g.nb_text);
  if (tiles == 0) return cudaSuccess;
  if (is_bf16) {
    if (g.D == 128) attn_simt_kernel<__nv_bfloat16, 128><<<tiles, kSimtWarps * 32, 0, st>>>(g, a);
    else attn_simt_kernel<__nv_bfloat16, 64><<<tiles, kSimtWarps * 32, 0, st>>>(g, a);
  } else {
    if (g.D == 128) attn_simt_kernel<float, 128><<<tiles, kSimtWarps * 32, 0, st>>>(g, a);
    else attn_simt_kernel<float, 64><<<tiles, kSimtWarps * 32, 0, st>>>(g, a);
  }
  return cudaGetLastError();
}

// ===========================================================================
// tcgen05 path (bf16, bs == 128)
//
// One CTA owns two query tiles (two consecutive tiles of the tile order).
// Warps 0-3 run the softmax of tile 0 and warps 4-7 that of tile 1, warp 8
// issues the TMA loads and warp 9 the MMAs.  While one softmax warpgroup
// works on its S, the tensor core runs the other tile's O += P V and its next
// S = Q K^T, so MMAs and exponentials overlap.  TMEM (512 columns): S of tile
// x at 128x, O of tile x at 256 + 128x; P (bf16 pairs, even key in the low
// half) overwrites the first 64 columns of S and is the A operand of the PV
// MMA.  K and V tiles stream through one ring of shared-memory slots in the
// order the MMA warp consumes them:
//   S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) PV1(1) S1(2) | ...
// A commit after S_x(s) covers every MMA issued before it, so when the
// softmax warps see S_x(s) the previous PV of the tile is complete and O_x
// may be rescaled in place.  The running max is only moved (and O rescaled)
// when it grows by more than 8 in log2 units; until then the exponentials
// are taken against the stale max (values stay below 2^8).
// ===========================================================================
template <int HD>
struct TcLayout {
  static constexpr int kTile = 128 * HD * 2;   // one 128-row bf16 tile
  static constexpr int kPanel = 128 * 128;     // 128 rows x 128 bytes (one TMA box)
  static constexpr int kStages = HD == 128 ? 4 : 8;
  static constexpr int kQ = 0;                 // two query tiles
  static constexpr int kRing = kQ + 2 * kTile; // K/V ring
  static constexpr int kBars = kRing + kStages * kTile;
  // q_full[2], kv_full[kStages], kv_empty[kStages], s_full[2], p_full[2], o_final[2], final
  static constexpr int kBarQ = 0, kBarFull = 2, kBarEmpty = 2 + kStages, kBarS = 2 + 2 * kStages,
                       kBarP = kBarS + 2, kBarO = kBarP + 2, kBarFinal = kBarO + 2;
  static constexpr int kNumBars = kBarFinal + 1;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

// Warps 0-3 and 4-7: softmax of tile 0 and tile 1; warp 8: TMA producer;
// warp 9: MMA issuer; warps 10-11 only complete the third warpgroup so that
// registers can be moved between warpgroups with setmaxnreg.
constexpr int kTcThreads = 384;
// Registers per thread: the launch gives every thread kRegsLaunch; then the
// producer/MMA warpgroup drops to kRegsSmall and the two softmax warpgroups
// rise to kRegsSoftmax.  2 * 128 * kRegsSoftmax + 128 * kRegsSmall must not
// exceed 384 * kRegsLaunch (checked below).
constexpr int kRegsLaunch = 168, kRegsSoftmax = 216, kRegsSmall = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsSmall <= kTcThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;      // log2 units

// Visits the MMA work of the two tiles in issue order: f(kind, tile, step),
// kind 0 = S = Q K^T (consumes a K slot), kind 1 = O += P V (a V slot).
// Stops early and returns false if f does.
template <class F>
__device__ __forceinline__ bool for_each_event(int n0, int n1, F&& f) {
  if (n0 > 0 && !f(0, 0, 0)) return false;
  if (n1 > 0 && !f(0, 1, 0)) return false;
  const int rounds = n0 > n1 ? n0 : n1;
  for (int r = 0; r < rounds; ++r) {
    if (r < n0) {
      if (!f(1, 0, r)) return false;
      if (r + 1 < n0 && !f(0, 0, r + 1)) return false;
    }
    if (r < n1) {
      if (!f(1, 1, r)) return false;
      if (r + 1 < n1 && !f(0, 1, r + 1)) return false;
    }
  }
  return true;
}

// Issues the TMA loads of one 128-row tile (Q, K or V of block j of head
// bh) into shared memory at dst, completing on bar.  Blocked layout: a 2D box
// of the block's contiguous rows.  Original layout (ORIG): a 5D box
// (d, head, x, y, t) whose shared-memory row order is the block's slot order
// (dt, dy, dx) and whose out-of-range part (the grid's padding) is zero-filled,
// or a 3D box (d, head, token) over the text tokens.
template <bool ORIG, int HD>
__device__ __forceinline__ void load_tile(const TileMaps& m, int which, const Geo& g,
                                          const AttnArgs& a, long long bh, int j, uint32_t dst,
                                          uint32_t bar) {
  constexpr int kPanel = 128 * 128;
  if (!ORIG) {
    const int row = (int)((bh * (g.nb + g.nb_text) + j) * 128);
    const CUtensorMap* map = which == 0 ? &m.q : (which == 1 ? &m.k : &m.v);
#pragma unroll
    for (int p = 0; p < HD / 64; ++p) tma_load_2d(dst + p * kPanel, map, 64 * p, row, bar);
  } else {
    // one batch element per launch: bh < Hd, so h = bh (kept general)
    const int h = (int)bh - (int)fdiv((uint32_t)bh, a.div_hd) * g.Hd;
    if (j < g.nb) {
      const int q1 = (int)fdiv((uint32_t)j, a.div_nbx), tb = (int)fdiv((uint32_t)q1, a.div_nby);
      const int xb = j - q1 * g.nbx, yb = q1 - tb * g.nby;
      const CUtensorMap* map = which == 0 ? &m.q : (which == 1 ? &m.k : &m.v);
#pragma unroll
      for (int p = 0; p < HD / 64; ++p)
        tma_load_5d(dst + p * kPanel, map, 64 * p, h, xb * g.bc, yb * g.br, tb * g.bf, bar);
    } else {
      const CUtensorMap* map = which == 0 ? &m.qt : (which == 1 ? &m.kt : &m.vt);
#pragma unroll
      for (int p = 0; p < HD / 64; ++p) tma_load_3d(dst + p * kPanel, map, 64 * p, h, (j - g.nb) * 128, bar);
    }
  }
}

template <int HD, bool ORIG>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(Geo g, AttnArgs a, const __grid_constant__ TileMaps maps) {
  using L = TcLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_addr(sm);
  const uint32_t sRing = sb + L::kRing;
  const uint32_t bar0 = sb + L::kBars;
  auto bar = [&](int x) { return bar0 + 8u * (uint32_t)x; };
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kAbort);
  const long long lim = a.wait_limit > 0 ? a.wait_limit : kWaitLimitDefault;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbk = g.nb + g.nb_text;
  const int n_tiles = map_count(a.map, g.B * g.Hd) * nbk;

  // The two query tiles of this CTA (held in scalars: a runtime-indexed array
  // would live in local memory), and how many leading steps they share.
  int i0 = -1, i1 = -1, n0 = 0, n1 = 0, c_shared = 0;
  int chunk = -1, kbase = 0;   // a text-chunk CTA of the paired schedule: its chunk and first key block
  long long bh0 = 0, bh1 = 0;
  const int32_t* list0;
  const int32_t* list1;
  if (a.pair_sched == nullptr) {
    int b, h, i;
    if (2 * (int)blockIdx.x < n_tiles) {
      decode_tile(g, a.map, 2 * blockIdx.x, b, h, i);
      i0 = i; bh0 = (long long)b * g.Hd + h; n0 = list_length(g, a, bh0, i);
    }
    if (2 * (int)blockIdx.x + 1 < n_tiles) {
      decode_tile(g, a.map, 2 * blockIdx.x + 1, b, h, i);
      i1 = i; bh1 = (long long)b * g.Hd + h; n1 = list_length(g, a, bh1, i);
    }
    list0 = a.idx + (bh0 * g.nb + (i0 >= 0 && i0 < g.nb ? i0 : 0)) * a.kmax;
    list1 = a.idx + (bh1 * g.nb + (i1 >= 0 && i1 < g.nb ? i1 : 0)) * a.kmax;
  } else {
    // Paired schedule, head-major: each head's group of CTAs opens with its
    // text pairs split into text_chunks key chunks (one CTA each, about as
    // long as a video pair), then its video pairs; entry (h, t) names the two
    // tiles and the shared count.  A text chunk reads its head's K / V while
    // the head's video pairs do, so one pass over K / V comes from DRAM.
    const int n_heads = map_count(a.map, g.B * g.Hd);
    (void)n_heads;
    const int vpairs = a.pairs_per_head - a.text_pairs;
    const int tp = a.text_pairs, nch = a.text_chunks, per = tp * nch + vpairs;
    const int m = (int)blockIdx.x / per;
    int t = (int)blockIdx.x % per;
    if (t < tp * nch) {
      chunk = t % nch;
      t = t / nch;
    } else {
      t = tp + (t - tp * nch);
    }
    const long long bh = map_bh(a.map, m);
    const long long ent = bh * a.pairs_per_head + t;
    const int4 se = __ldg(reinterpret_cast<const int4*>(a.pair_sched) + ent);
    bh0 = bh1 = bh;
    i0 = se.x;
    i1 = se.y;
    if (chunk >= 0) {
      // key blocks [chunk * len, ...) of the dense text rows, shared by both tiles
      kbase = chunk * a.text_chunk_len;
      const int len = min(a.text_chunk_len, nbk - kbase);
      n0 = i0 >= 0 ? len : 0;
      n1 = i1 >= 0 ? len : 0;
      c_shared = min(n0, n1);   // a single-tile pair (odd text block count) shares nothing
    } else {
      if (i0 >= 0) n0 = list_length(g, a, bh, i0);
      if (i1 >= 0) n1 = list_length(g, a, bh, i1);
      c_shared = min(se.z, min(n0, n1));
    }
    list0 = a.pair_lists + (ent * 2 + 0) * a.kmax;
    list1 = a.pair_lists + (ent * 2 + 1) * a.kmax;
  }
  // Key block of step s of tile x; -1 for an out-of-range list entry.
  auto block_at = [&](int x, int s) -> int {
    const int i = x ? i1 : i0;
    const int j = i >= g.nb ? kbase + s : __ldg((x ? list1 : list0) + s);
    return (j >= 0 && j < nbk) ? j : -1;
  };

  if (threadIdx.x == 0) {
    for (int x = 0; x < L::kNumBars; ++x)
      mbar_init(bar(x), (x == L::kBarP || x == L::kBarP + 1) ? 128u : 1u);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sb + L::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::kTmemSlot);
  constexpr uint32_t kTileBytes = L::kTile;
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, HD, 0, 1);
  if (warp >= 8) {
   // ============================================================ warpgroup 2
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSmall));
   if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int x = 0; x < 2; ++x) {
        if ((x ? n1 : n0) == 0) continue;
        mbar_arrive_expect_tx(bar(L::kBarQ + x), kTileBytes);
        load_tile<ORIG, HD>(maps, 0, g, a, x ? bh1 : bh0, x ? i1 : i0, sb + L::kQ + x * kTileBytes,
                            bar(L::kBarQ + x));
      }
      int pos = 0;
      bool bad = false;
      for_each_event(n0, n1, [&](int kind, int x, int s) -> bool {
        // tile 1's first c_shared steps use the K / V tiles tile 0 fetched
        if (x == 1 && s < c_shared) return true;
        int j = block_at(x, s);
        if (j < 0) { bad = true; j = 0; }   // load some tile; the softmax masks the step
        // test hook: a copy that never lands, so that the consumer's wait runs out
        if (pos + 1 == a.hold_load && blockIdx.x == 0) return false;
        const int slot = pos % L::kStages;
        if (pos >= L::kStages &&
            !mbar_wait(bar(L::kBarEmpty + slot), ((pos / L::kStages) - 1) & 1, abort, lim))
          return false;
        const uint32_t dst = sRing + slot * kTileBytes;
        mbar_arrive_expect_tx(bar(L::kBarFull + slot), kTileBytes);
        load_tile<ORIG, HD>(maps, kind == 0 ? 1 : 2, g, a, x ? bh1 : bh0, j, dst, bar(L::kBarFull + slot));
        ++pos;
        return true;
      });
      if (bad) set_status(a.status, 6);
      // Never leave the CTA with a copy in flight: wait for the Q tiles and
      // the last kStages K/V copies issued (each slot's latest copy), also
      // after an abort (these waits ignore it; issued copies always land).
      for (int x = 0; x < 2; ++x)
        if ((x ? n1 : n0) > 0) mbar_wait_drain(bar(L::kBarQ + x), 0, lim);
      for (int p = (pos > L::kStages ? pos - L::kStages : 0); p < pos; ++p)
        mbar_wait_drain(bar(L::kBarFull + p % L::kStages), (p / L::kStages) & 1, lim);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int x = 0; x < 2; ++x)
        if ((x ? n1 : n0) > 0 && !mbar_wait(bar(L::kBarQ + x), 0, abort, lim)) ok = false;
      tc_fence_after();
      int pos = 0;
      int shared_slot[2] = {0, 0};   // ring slot of tile 0's K (S) and V (PV) of a shared step
      if (ok) {
        for_each_event(n0, n1, [&](int kind, int x, int s) -> bool {
          // a shared step: tile 0 (issued first) waits for the tile and keeps
          // it; tile 1 reuses it and releases it
          const bool shared = s < c_shared;
          int slot;
          if (shared && x == 1) {
            slot = kind == 0 ? shared_slot[0] : shared_slot[1];
          } else {
            slot = pos % L::kStages;
            if (!mbar_wait(bar(L::kBarFull + slot), (pos / L::kStages) & 1, abort, lim)) return false;
            tc_fence_after();
            ++pos;
            if (shared) {
              if (kind == 0) shared_slot[0] = slot;
              else shared_slot[1] = slot;
            }
          }
          const uint32_t src = sRing + slot * kTileBytes;
          const uint32_t tS = tmem + 128u * x;
          if (kind == 0) {
            const uint32_t sQ = sb + L::kQ + x * kTileBytes;
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
              const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
              mma_bf16_ss(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(src + off, 16, 1024),
                          idesc_s, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar(L::kBarS + x));
          } else {
            if (!mbar_wait(bar(L::kBarP + x), s & 1, abort, lim)) return false;
            tc_fence_after();
            const uint32_t tO = tmem + 256u + 128u * x;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16_ts(tO, tS + 8u * kk, smem_desc_sw128(src + kk * 2048, L::kPanel, 1024), idesc_o,
                          (s > 0 || kk > 0) ? 1u : 0u);
            if (s == (x ? n1 : n0) - 1) tc_commit(bar(L::kBarO + x));
          }
          if (!(shared && x == 0)) tc_commit(bar(L::kBarEmpty + slot));
          return true;
        });
      }
      // Every MMA issued must be complete before TMEM is released, also
      // after an abort (the commit tracks all of them; the wait ignores abort).
      tc_commit(bar(L::kBarFinal));
      mbar_wait_drain(bar(L::kBarFinal), 0, lim);
    }
   }
  } else {
    // ============================================================ warpgroups 0-1
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax warpgroups
    const int x = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;                        // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + 128u * x + lane_off;
    const uint32_t tO = tmem + 256u + 128u * x + lane_off;
    const int n = x ? n1 : n0;
    const int qi = x ? i1 : i0;
    const long long qbh = x ? bh1 : bh0;
    if (qi >= 0) {
      float m_run = -INFINITY, l = 0.f;
      bool ok = true;
      // Block id and slot-validity mask of the next step, loaded one step
      // ahead so that their latency hides behind the wait for S.
      int j_next = n > 0 ? block_at(x, 0) : -1;
      uint4 mw_next = j_next >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.masks) + j_next)
                                  : make_uint4(0u, 0u, 0u, 0u);
      for (int s = 0; s < n; ++s) {
        const uint4 mw = mw_next;
        if (s + 1 < n) {
          j_next = block_at(x, s + 1);
          mw_next = j_next >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.masks) + j_next)
                                : make_uint4(0u, 0u, 0u, 0u);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::kBarS + x), s & 1, abort, lim))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        TMEM_LD32(tS + 0, (sr + 0));
        TMEM_LD32(tS + 32, (sr + 32));
        TMEM_LD32(tS + 64, (sr + 64));
        TMEM_LD32(tS + 96, (sr + 96));
        TMEM_LD_WAIT((sr + 0));
        TMEM_LD_WAIT((sr + 32));
        TMEM_LD_WAIT((sr + 64));
        TMEM_LD_WAIT((sr + 96));
        if ((mw.x & mw.y & mw.z & mw.w) != 0xffffffffu) {
          const uint32_t w4[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((w4[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
        }
        // Row max over 8 independent partial maxima (short dependency chains).
        float mp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = __uint_as_float(sr[k]);
#pragma unroll
        for (int c = 8; c < 128; ++c) mp[c & 7] = fmaxf(mp[c & 7], __uint_as_float(sr[c]));
        const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                               fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        const float m_cand = mx * a.scale_log2;
        const bool need = m_cand > m_run + kRescaleThreshold;
        const bool any_need = __any_sync(0xffffffffu, need);
        float scale = 1.f;
        if (any_need) {
          const float m_new = need ? m_cand : m_run;
          scale = need ? fast_ex2(m_run - m_new) : 1.f;
          l *= scale;
          m_run = m_new;
        }
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
        const float2 neg_m = make_float2(-m_use, -m_use);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float2 t = fma2(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])),
                                sl2, neg_m);
          const float2 p = make_float2(fast_ex2(t.x), fast_ex2(t.y));
          acc[c & 3] = add2(acc[c & 3], p);
          pk[c] = pack_bf16x2(p.x, p.y);
        }
        const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
        const float2 a03 = add2(a01, a23);
        l += a03.x + a03.y;
        TMEM_ST32(tS + 0, (pk + 0));
        TMEM_ST32(tS + 32, (pk + 32));
        // O of the previous steps is complete (this S was committed after the
        // previous PV), so it can be rescaled before this step's PV is issued.
        if (any_need && s > 0) {
#pragma unroll
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t orr[32];
            TMEM_LD32(tO + c0, orr);
            TMEM_LD_WAIT(orr);
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * scale);
            TMEM_ST32(tO + c0, orr);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::kBarP + x));
      }
      // ---- epilogue: O / l -> blocked output row
      if (ok && n > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarO + x), 0, abort, lim));
        tc_fence_after();
      }
      if (chunk >= 0) {
        // Text chunk: the unnormalised O row, the running max (log2 units)
        // and the row sum go to the partial buffer; the merge pass combines
        // the chunks of each text row.
        const bool okr = ok && n > 0;
        float* prow = a.part + ((((long long)qbh * g.nb_text + (qi - g.nb)) * a.text_chunks + chunk) * 128 + r) *
                                   (long long)(HD + 4);
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t orr[32];
          if (okr) {
            TMEM_LD32(tO + c0, orr);
            TMEM_LD_WAIT(orr);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = 0u;
          }
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            reinterpret_cast<uint4*>(prow + c0)[c4] =
                make_uint4(orr[4 * c4], orr[4 * c4 + 1], orr[4 * c4 + 2], orr[4 * c4 + 3]);
        }
        // an aborted CTA marks its rows (sum -1): the merge writes them as zeros
        *reinterpret_cast<float4*>(prow + HD) =
            make_float4(okr ? m_run : -INFINITY, okr ? l : -1.f, 0.f, 0.f);
      } else {
        const uint4 qm = __ldg(reinterpret_cast<const uint4*>(a.masks) + qi);
        const uint32_t qw4[4] = {qm.x, qm.y, qm.z, qm.w};
        const bool slot_real = (qw4[r >> 5] >> (r & 31)) & 1u;
        const bool row_valid = slot_real && ok && n > 0;
        const float inv = (row_valid && l > 0.f) ? 1.f / l : 0.f;
        // Blocked layout: every slot row is written (pad rows 0).  Original
        // layout: each real slot's row goes to its token, pad slots are dropped.
        long long orow_idx;
        if (!ORIG) {
          orow_idx = (qbh * nbk + qi) * 128 + r;
        } else {
          const long long tok = slot_token(g, qi, r);
          orow_idx = tok >= 0 ? tok * g.Hd + (qbh % g.Hd) : -1;
        }
        uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + (orow_idx < 0 ? 0 : orow_idx) * HD);
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t orr[32];
          if (ok && n > 0) {
            TMEM_LD32(tO + c0, orr);
            TMEM_LD_WAIT(orr);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = 0u;
          }
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(orr[8 * c8 + 0]) * inv, __uint_as_float(orr[8 * c8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(orr[8 * c8 + 2]) * inv, __uint_as_float(orr[8 * c8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(orr[8 * c8 + 4]) * inv, __uint_as_float(orr[8 * c8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(orr[8 * c8 + 6]) * inv, __uint_as_float(orr[8 * c8 + 7]) * inv);
            if (orow_idx >= 0) orow[c0 / 8 + c8] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort) set_status(a.status, 4);
}

size_t attn_tc_smem_bytes(int D) {
  return D == 128 ? TcLayout<128>::kAlloc : TcLayout<64>::kAlloc;
}

template <int HD, bool ORIG>
static cudaError_t launch_tc_t(const Geo& g, const AttnArgs& a, const TileMaps& maps, int ctas,
                               cudaStream_t st) {
  // The setmaxnreg split assumes the launch gives every thread exactly
  // kRegsLaunch registers; refuse to launch a build where that is not so.
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, attn_tc_kernel<HD, ORIG>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  const int smem = TcLayout<HD>::kAlloc;
  e = cudaFuncSetAttribute(attn_tc_kernel<HD, ORIG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<HD, ORIG><<<ctas, kTcThreads, smem, st>>>(g, a, maps);
  return cudaGetLastError();
}

// Blocked layout in and out (bsa_attention).
cudaError_t launch_attn_tc(const Geo& g, const AttnArgs& a, const TileMaps& maps, cudaStream_t st) {
  const int tiles = map_count(a.map, g.B * g.Hd) * (g.nb + g.nb_text);
  if (tiles == 0) return cudaSuccess;
  const int ctas = (tiles + 1) / 2;
  return g.D == 128 ? launch_tc_t<128, false>(g, a, maps, ctas, st)
                    : launch_tc_t<64, false>(g, a, maps, ctas, st);
}

// Original layout in and out, one batch element (g.B == 1): the layout
// transform and its inverse happen inside the loads and the epilogue.
cudaError_t launch_attn_tc_orig(const Geo& g, const AttnArgs& a, const TileMaps& maps,
                                cudaStream_t st) {
  const int tiles = map_count(a.map, g.Hd) * (g.nb + g.nb_text);
  if (tiles == 0 || g.B != 1) return g.B != 1 ? cudaErrorInvalidValue : cudaSuccess;
  // paired schedule: one CTA per video pair (a head with an odd tile count
  // has a single-tile entry) and per key chunk of each text pair
  const int ctas = a.pair_sched ? map_count(a.map, g.Hd) *
                                      (a.pairs_per_head - a.text_pairs + a.text_pairs * a.text_chunks)
                                : (tiles + 1) / 2;
  return g.D == 128 ? launch_tc_t<128, true>(g, a, maps, ctas, st)
                    : launch_tc_t<64, true>(g, a, maps, ctas, st);
}

// Merge of the key-chunk partials of the text rows (SPADE §3.3 (3)'s online
// softmax, finished across chunks): for a row with partials (O_c, m_c, l_c),
// M = max_c m_c, w_c = 2^(m_c - M), output = sum_c w_c O_c / sum_c w_c l_c,
// rounded to bf16 (the same quotient the one-CTA path forms, with the sums
// regrouped).  One warp per text row, lanes over the head dimension.
constexpr int kMergeWarps = 8;

template <int HD>
__global__ void __launch_bounds__(kMergeWarps * 32) text_merge_kernel(Geo g, MergeArgs a) {
  constexpr int kPer = HD / 32;                       // columns per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long u = (long long)blockIdx.x * kMergeWarps + warp;   // text token
  if (u >= g.n_text) return;
  const long long bh = map_bh(a.map, blockIdx.y);
  const int tb = (int)(u / 128), r = (int)(u % 128);
  const long long stride_c = 128ll * (HD + 4);
  const float* base = a.part + (((bh * g.nb_text + tb) * a.text_chunks) * 128 + r) * (long long)(HD + 4);
  float M = -INFINITY;
  for (int c = 0; c < a.text_chunks; ++c) M = fmaxf(M, base[c * stride_c + HD]);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float lsum = 0.f;
  bool aborted = false;
  for (int c = 0; c < a.text_chunks; ++c) {
    const float* pc = base + c * stride_c;
    const float mc = pc[HD];
    aborted = aborted || pc[HD + 1] < 0.f;
    const float w = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
    lsum = fmaf(w, pc[HD + 1], lsum);
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, pc[kPer * lane + e], acc[e]);
  }
  const float inv = (lsum > 0.f && !aborted) ? 1.f / lsum : 0.f;
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) +
                        ((g.n_video + u) * g.Hd + (bh % g.Hd)) * HD + kPer * lane;
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

cudaError_t launch_text_merge(const Geo& g, const MergeArgs& a, cudaStream_t st) {
  const int heads = map_count(a.map, g.Hd);
  if (g.n_text == 0 || heads == 0 || g.B != 1) return g.B != 1 ? cudaErrorInvalidValue : cudaSuccess;
  const dim3 grid((unsigned)((g.n_text + kMergeWarps - 1) / kMergeWarps), (unsigned)heads);
  if (g.D == 128) text_merge_kernel<128><<<grid, kMergeWarps * 32, 0, st>>>(g, a);
  else text_merge_kernel<64><<<grid, kMergeWarps * 32, 0, st>>>(g, a);
  return cudaGetLastError();
}

}  // namespace bsa
