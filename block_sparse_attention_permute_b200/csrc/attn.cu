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
//  * attn_tc_kernel (bf16, 128-token blocks, D in {64,128}): one CTA per
//    (batch, head, query block).  Warp 4 issues TMA loads of Q once and of
//    the K/V tiles of the selected key blocks only (two stages); warp 5 issues
//    tcgen05.mma: S = Q K^T into TMEM, O += P V into TMEM; warps 0-3 own one
//    query row per thread: they read S from TMEM, apply the pad mask and the
//    online softmax (exp2 of log2e-prescaled logits, fp32 statistics),
//    rescale O in TMEM when the running max grows, and write P (bf16) to
//    shared memory for the PV product.  The epilogue divides by the row sum.
//  * attn_simt_kernel (any dtype, any block size <= 256): one warp per query
//    row, fp32 scores and online softmax, exact fp32 arithmetic.  It serves
//    fp32 inputs and block shapes the tensor-core path does not take.
// Text query blocks (ids >= nb) attend every key block.
#include "kernels.cuh"

namespace bsa {


// Tile order: text query tiles first (they have the longest lists), then the
// video tiles, head-major so that one head's K/V stays resident in L2.
__device__ __forceinline__ void decode_tile(const Geo& g, int L, int& b, int& h, int& i) {
  const int n_text_tiles = g.B * g.Hd * g.nb_text;
  if (L < n_text_tiles) {
    i = g.nb + L % g.nb_text;
    const int bh = L / g.nb_text;
    h = bh % g.Hd;
    b = bh / g.Hd;
  } else {
    L -= n_text_tiles;
    i = L % g.nb;
    const int bh = L / g.nb;
    h = bh % g.Hd;
    b = bh / g.Hd;
  }
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
  decode_tile(g, blockIdx.x, b, h, i);
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
  const int tiles = g.B * g.Hd * (g.nb + g.nb_text);
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
// ===========================================================================
template <int HD>
struct TcLayout {
  static constexpr int kTile = 128 * HD * 2;   // one 128-row bf16 tile
  static constexpr int kPanel = 128 * 128;     // 128 rows x 128 bytes (one TMA box)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;        // 2 stages
  static constexpr int kV = kK + 2 * kTile;    // 2 stages
  static constexpr int kP = kV + 2 * kTile;    // 128 x 128 bf16, 2 panels
  static constexpr int kBars = kP + 2 * kPanel;
  // 0 q_full, 1-2 k_full, 3-4 v_full, 5-6 kv_empty, 7 s_full, 8 p_full, 9 o_done, 10 final
  static constexpr int kNumBars = 11;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

constexpr int kTcThreads = 192;
constexpr uint32_t kTmemCols = 256;

template <int HD>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(Geo g, AttnArgs a, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  using L = TcLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_addr(sm);
  const uint32_t sQ = sb + L::kQ, sK = sb + L::kK, sV = sb + L::kV, sP = sb + L::kP;
  const uint32_t bar0 = sb + L::kBars;
  const uint32_t bar_q = bar0, bar_s = bar0 + 7 * 8, bar_p = bar0 + 8 * 8, bar_o = bar0 + 9 * 8;
  const uint32_t bar_final = bar0 + 10 * 8;
  auto bar_k = [&](int st) { return bar0 + (1 + st) * 8; };
  auto bar_v = [&](int st) { return bar0 + (3 + st) * 8; };
  auto bar_e = [&](int st) { return bar0 + (5 + st) * 8; };
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, h, i;
  decode_tile(g, blockIdx.x, b, h, i);
  const long long bh = (long long)b * g.Hd + h;
  const int nbk = g.nb + g.nb_text;
  const bool dense_row = i >= g.nb;
  const int n = list_length(g, a, bh, i);
  const int32_t* list = a.idx + (bh * g.nb + (dense_row ? 0 : i)) * a.kmax;
  auto block_at = [&](int s) -> int {
    const int j = dense_row ? s : __ldg(list + s);
    return (j >= 0 && j < nbk) ? j : -1;
  };

  if (threadIdx.x == 0) {
    for (int x = 0; x < L::kNumBars; ++x) mbar_init(bar0 + 8 * x, x == 8 ? 128 : 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(sb + L::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::kTmemSlot);
  const uint32_t tS = tmem, tO = tmem + 128;
  constexpr uint32_t kTileBytes = L::kTile;
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, HD, 0, 1);

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int qrow = (int)((bh * nbk + i) * 128);
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      for (int p = 0; p < HD / 64; ++p) tma_load_2d(sQ + p * L::kPanel, &tq, 64 * p, qrow, bar_q);
      int it = 0;
      bool bad = false;
      for (int s = 0; s < n; ++s) {
        const int j = block_at(s);
        if (j < 0) { bad = true; continue; }
        const int st = it & 1;
        if (it >= 2 && !mbar_wait(bar_e(st), ((it >> 1) - 1) & 1, abort)) break;
        const int krow = (int)((bh * nbk + j) * 128);
        mbar_arrive_expect_tx(bar_k(st), kTileBytes);
        for (int p = 0; p < HD / 64; ++p)
          tma_load_2d(sK + st * kTileBytes + p * L::kPanel, &tk, 64 * p, krow, bar_k(st));
        mbar_arrive_expect_tx(bar_v(st), kTileBytes);
        for (int p = 0; p < HD / 64; ++p)
          tma_load_2d(sV + st * kTileBytes + p * L::kPanel, &tv, 64 * p, krow, bar_v(st));
        ++it;
      }
      if (bad) set_status(a.status, 6);
      // Never leave the CTA with a copy in flight: wait for the last loads.
      mbar_wait(bar_q, 0, abort);
      for (int x = (it >= 2 ? it - 2 : 0); x < it; ++x) {
        mbar_wait(bar_k(x & 1), (x >> 1) & 1, abort);
        mbar_wait(bar_v(x & 1), (x >> 1) & 1, abort);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0;
      bool ok = mbar_wait(bar_q, 0, abort);
      tc_fence_after();
      auto issue_pv = [&](int x) -> bool {
        const int st = x & 1;
        if (!mbar_wait(bar_p, x & 1, abort)) return false;
        if (!mbar_wait(bar_v(st), (x >> 1) & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc_sw128(sP + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sV + st * kTileBytes + kk * 2048, L::kPanel, 1024);
          mma_bf16_ss(tO, ad, bd, idesc_o, (x > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar_o);
        tc_commit(bar_e(st));
        return true;
      };
      for (int s = 0; s < n && ok; ++s) {
        if (block_at(s) < 0) continue;
        const int st = it & 1;
        if (!mbar_wait(bar_k(st), (it >> 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        if (it > 0 && !issue_pv(it - 1)) { ok = false; break; }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sQ + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + st * kTileBytes + off, 16, 1024);
          mma_bf16_ss(tS, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_s);
        ++it;
      }
      if (ok && it > 0) issue_pv(it - 1);
      // Every MMA issued must be complete before TMEM is released.
      tc_commit(bar_final);
      mbar_wait(bar_final, 0, abort);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = warp * 32 + lane;                      // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    int it = 0;
    bool ok = true;
    for (int s = 0; s < n; ++s) {
      const int j = block_at(s);
      if (j < 0) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s, it & 1, abort))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      TMEM_LD32(tS + lane_off + 0, (sr + 0));
      TMEM_LD32(tS + lane_off + 32, (sr + 32));
      TMEM_LD32(tS + lane_off + 64, (sr + 64));
      TMEM_LD32(tS + lane_off + 96, (sr + 96));
      TMEM_LD_WAIT((sr + 0));
      TMEM_LD_WAIT((sr + 32));
      TMEM_LD_WAIT((sr + 64));
      TMEM_LD_WAIT((sr + 96));
      const uint4 mw = __ldg(reinterpret_cast<const uint4*>(a.masks) + j);
      if ((mw.x & mw.y & mw.z & mw.w) != 0xffffffffu) {
        const uint32_t w4[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!((w4[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      const float m_new = fmaxf(m, mx * a.scale_log2);
      const float corr = fast_ex2(m - m_new);
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float p = fast_ex2(fmaf(__uint_as_float(sr[c]), a.scale_log2, -m_new));
        rowsum += p;
        sr[c] = __float_as_uint(p);
      }
      l = l * corr + rowsum;
      m = m_new;
      if (it > 0) {
        // PV of the previous step must be done: P buffer free, O stable.
        if (!__all_sync(0xffffffffu, mbar_wait(bar_o, (it - 1) & 1, abort))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t orr[32];
            TMEM_LD32(tO + lane_off + c0, orr);
            TMEM_LD_WAIT(orr);
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * corr);
            TMEM_ST32(tO + lane_off + c0, orr);
          }
          tmem_st_wait();
        }
      }
      // P row -> shared memory, K-major with the 128-byte swizzle.
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(sr[8 * c8 + 0]), __uint_as_float(sr[8 * c8 + 1]));
        v.y = pack_bf16x2(__uint_as_float(sr[8 * c8 + 2]), __uint_as_float(sr[8 * c8 + 3]));
        v.z = pack_bf16x2(__uint_as_float(sr[8 * c8 + 4]), __uint_as_float(sr[8 * c8 + 5]));
        v.w = pack_bf16x2(__uint_as_float(sr[8 * c8 + 6]), __uint_as_float(sr[8 * c8 + 7]));
        const uint32_t addr = sP + (c8 >> 3) * L::kPanel + r * 128 + ((((c8 & 7) ^ (r & 7))) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                     "r"(v.z), "r"(v.w)
                     : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p);
      ++it;
    }
    // ---- epilogue: O / l -> blocked output row
    if (ok && it > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (it - 1) & 1, abort));
      tc_fence_after();
    }
    const uint4 qm = __ldg(reinterpret_cast<const uint4*>(a.masks) + i);
    const uint32_t qw4[4] = {qm.x, qm.y, qm.z, qm.w};
    const bool row_valid = ((qw4[r >> 5] >> (r & 31)) & 1u) && ok && it > 0;
    const float inv = (row_valid && l > 0.f) ? 1.f / l : 0.f;
    uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) +
                                           ((bh * nbk + i) * 128 + r) * HD);
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += 32) {
      uint32_t orr[32];
      if (ok && it > 0) {
        TMEM_LD32(tO + lane_off + c0, orr);
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
        orow[c0 / 8 + c8] = v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort) set_status(a.status, 4);
}

size_t attn_tc_smem_bytes(int D) {
  return D == 128 ? TcLayout<128>::kAlloc : TcLayout<64>::kAlloc;
}

cudaError_t launch_attn_tc(const Geo& g, const AttnArgs& a, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  const int tiles = g.B * g.Hd * (g.nb + g.nb_text);
  if (tiles == 0) return cudaSuccess;
  cudaError_t e;
  if (g.D == 128) {
    const int smem = TcLayout<128>::kAlloc;
    e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<128><<<tiles, kTcThreads, smem, st>>>(g, a, tq, tk, tv);
  } else {
    const int smem = TcLayout<64>::kAlloc;
    e = cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<64><<<tiles, kTcThreads, smem, st>>>(g, a, tq, tk, tv);
  }
  return cudaGetLastError();
}

}  // namespace bsa
