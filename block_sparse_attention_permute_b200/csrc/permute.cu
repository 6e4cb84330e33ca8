// permute.cu — layout transform between the original token order and the
// block-contiguous order, fused with the mean summarizer.
//
// SPADE (arXiv 2608.03335) §3.3: "Q, K, V are first rearranged into a blocked
// layout by the Selected Blocking Scheme for intra-block contiguity. The
// Summarizer Expression then produces one vector per Q/K block"; "(1) Operator
// fusion. We fuse layout transform (blocking), summarization ... into one CUDA
// kernel".  Block shapes are frames x rows x cols (DecoupAttn Plans README,
// "Contents").
//
// One CTA moves one (tensor, batch, head, block) tile: bs rows of D elements.
// Every row is moved as 16-byte vectors (D=128 bf16: 16 vectors, so a warp
// covers two 256-byte rows per instruction).  The slot -> token map of the
// block is decoded once into shared memory.  HBM-bound: each byte is read
// once and written once.
#include <cmath>

#include "kernels.cuh"

namespace bsa {

enum GatherMode { kPermute = 0, kUnpermute = 1, kPool = 2, kPoolOrig = 3 };


constexpr int kGatherThreads = 256;
constexpr int kUnroll = 4;

template <typename T>
__device__ __forceinline__ void accumulate_vec(float* acc, const uint4& v) {
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(p[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  } else {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
}

template <typename T>
__device__ __forceinline__ void to_float(const uint4& v, float* f) {
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(p[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  } else {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
}

// One CTA's work: tile (tensor, b, h, block j).  With a.sics[tensor] set it
// also evaluates the intra-block estimator of SPADE §3.2, Eq. (4), the sum of
// all pairwise cosine similarities of the block's valid rows, in the form
// || sum_a q_a / |q_a| ||^2 (equal to Eq. (4) by expanding the square; a zero
// row has no direction and contributes nothing).  The running sum of unit
// rows is the r of the online form (Eq. (5)); squaring it once at the end
// instead of accumulating the cross terms keeps every term of the fp32 sum
// non-negative.
template <typename T, int D, int MODE, bool EXTRAS>
__device__ __forceinline__ void gather_block(const Geo& g, const void* src_ptr, void* dst_ptr,
                                             float* cent_ptr, float* sics_ptr, float* box_ptr,
                                             int j, int h, int b) {
  constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte vector
  constexpr int V = D / E;                // vectors per row
  constexpr int R = kGatherThreads / V;   // rows per pass
  __shared__ int s_tok[256];
  __shared__ float s_red[R * D];
  __shared__ float s_warp[kGatherThreads / 32];

  const int tid = threadIdx.x, row0 = tid / V, vec = tid % V;

  for (int s = tid; s < g.bs; s += kGatherThreads) s_tok[s] = (int)slot_token(g, j, s);
  __syncthreads();

  const long long blk_row0 = (long long)(b * g.Hd + h) * g.npad_tot + (long long)j * g.bs;
  const long long tok_base = (long long)b * g.n_tot;
  float* cent = (MODE != kUnpermute && j < g.nb) ? cent_ptr : nullptr;
  // SICS and box outputs exist only in the EXTRAS instances, which keeps
  // the plain copy / centroid instances lean (registers, occupancy).
  float* sics = (EXTRAS && MODE != kUnpermute && j < g.nb) ? sics_ptr : nullptr;
  float* box = (EXTRAS && MODE != kUnpermute && j < g.nb) ? box_ptr : nullptr;
  float acc[E], racc[E], vmax[E], vmin[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    acc[e] = racc[e] = 0.f;
    vmax[e] = -INFINITY;
    vmin[e] = INFINITY;
  }

  const uint4* src = reinterpret_cast<const uint4*>(src_ptr);
  uint4* dst = reinterpret_cast<uint4*>(dst_ptr);
  for (int s0 = 0; s0 < g.bs; s0 += R * kUnroll) {
    uint4 buf[kUnroll];
    int tok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = s0 + u * R + row0;
      tok[u] = s < g.bs ? s_tok[s] : -2;
      buf[u] = make_uint4(0, 0, 0, 0);
      if (tok[u] >= 0) {
        const long long vi = (MODE == kPermute || MODE == kPoolOrig)
                                 ? ((tok_base + tok[u]) * g.Hd + h) * V + vec
                                 : (blk_row0 + s) * V + vec;
        buf[u] = __ldg(src + vi);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = s0 + u * R + row0;
      if (MODE == kPermute && tok[u] >= -1) dst[(blk_row0 + s) * V + vec] = buf[u];
      if (MODE == kUnpermute && tok[u] >= 0) dst[((tok_base + tok[u]) * g.Hd + h) * V + vec] = buf[u];
      if (MODE != kUnpermute && cent != nullptr && tok[u] >= 0) accumulate_vec<T>(acc, buf[u]);
      if (EXTRAS && MODE != kUnpermute && box != nullptr && tok[u] >= 0) {
        float f[E];
        to_float<T>(buf[u], f);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          vmax[e] = fmaxf(vmax[e], f[e]);
          vmin[e] = fminf(vmin[e], f[e]);
        }
      }
      if (EXTRAS && MODE != kUnpermute && sics != nullptr) {
        // Every lane takes part (pad and out-of-range rows hold zeros): the V
        // lanes of one row are an aligned group of the warp.
        float f[E], ss = 0.f;
        to_float<T>(buf[u], f);
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
        for (int o = V / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) racc[e] = fmaf(f[e], inv, racc[e]);
      }
    }
  }

  if (MODE != kUnpermute && cent != nullptr) {
#pragma unroll
    for (int e = 0; e < E; ++e) s_red[row0 * D + vec * E + e] = acc[e];
    __syncthreads();
    if (tid < D) {
      float sum = 0.f;
      for (int r = 0; r < R; ++r) sum += s_red[r * D + tid];
      const float n = (float)block_valid_count(g, j);
      cent[((long long)(b * g.Hd + h) * g.nb + j) * D + tid] = sum / n;
    }
  }

  if (EXTRAS && MODE != kUnpermute && box != nullptr) {
    // per dimension: max, then min, over the R row groups (exact in fp32)
    float* out = box + ((long long)(b * g.Hd + h) * g.nb + j) * D * 2;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      __syncthreads();  // s_red is reused
#pragma unroll
      for (int e = 0; e < E; ++e) s_red[row0 * D + vec * E + e] = pass == 0 ? vmax[e] : vmin[e];
      __syncthreads();
      if (tid < D) {
        float r = s_red[tid];
        for (int rr = 1; rr < R; ++rr)
          r = pass == 0 ? fmaxf(r, s_red[rr * D + tid]) : fminf(r, s_red[rr * D + tid]);
        out[2 * tid + pass] = r;
      }
    }
  }

  if (EXTRAS && MODE != kUnpermute && sics != nullptr) {
    __syncthreads();  // s_red is reused after the centroid reduction
#pragma unroll
    for (int e = 0; e < E; ++e) s_red[row0 * D + vec * E + e] = racc[e];
    __syncthreads();
    float r2 = 0.f;
    if (tid < D) {
      float r = 0.f;
      for (int rr = 0; rr < R; ++rr) r += s_red[rr * D + tid];
      r2 = r * r;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, o);
    if ((tid & 31) == 0) s_warp[tid >> 5] = r2;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < D / 32; ++w) t += s_warp[w];
      sics[(long long)(b * g.Hd + h) * g.nb + j] = t;
    }
  }
}

template <typename T, int D, int MODE, bool EXTRAS>
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(Geo g, GatherArgs a) {
  // Constant-index reads of the pointer arrays (a dynamic index would copy
  // the argument block to local memory).
  const int t = a.map.n ? (int)blockIdx.z : (int)(blockIdx.z % a.ntensors);
  const int bh = a.map.n ? (int)a.map.bh[blockIdx.y] : (int)(blockIdx.z / a.ntensors) * g.Hd + (int)blockIdx.y;
  const void* src = t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2];
  void* dst = t == 0 ? a.dst[0] : t == 1 ? a.dst[1] : a.dst[2];
  float* cent = t == 0 ? a.cent[0] : t == 1 ? a.cent[1] : a.cent[2];
  float* sics = t == 0 ? a.sics[0] : t == 1 ? a.sics[1] : a.sics[2];
  float* box = t == 0 ? a.box[0] : t == 1 ? a.box[1] : a.box[2];
  gather_block<T, D, MODE, EXTRAS>(g, src, dst, cent, sics, box, blockIdx.x, bh % g.Hd, bh / g.Hd);
}

// Centroids of the video blocks from the original layout, bf16 plans with
// 128-token blocks (the summarizer pass of bsa_forward).  One CTA of 128
// threads per (tensor, block j, group of heads); thread (head, v) owns the
// 16-byte column v of one head and streams it through the block's 128 slots,
// so a warp reads whole runs of adjacent heads of one token and no partial
// sums cross threads (M = 128 / R independent 16-byte loads per row group).  The sums are formed in the order of gather_block's
// kPool path (row group r = s mod R holds s = r, r + R, ...; the groups are
// then added in ascending r), so the centroids are bit-identical to the
// blocked-layout pool.
constexpr int kColThreads = 128;

// THREADS / V heads per CTA (the launcher picks the count that fills the
// GPU's CTA slots best); a thread's sum is the same for every count.
template <int D, int THREADS>
__global__ void __launch_bounds__(THREADS) pool_cols_kernel(Geo g, GatherArgs a) {
  using T = __nv_bfloat16;
  constexpr int E = 8;                      // bf16 elements per 16-byte vector
  constexpr int V = D / E;                  // vectors per row
  constexpr int R = kGatherThreads / V;     // row groups, as in gather_block
  constexpr int M = 128 / R;                // rows per group
  constexpr int HG = THREADS / V;           // heads per CTA
  __shared__ int s_tok[128];
  const int j = blockIdx.x, t = blockIdx.z;
  const int p = blockIdx.y * HG + (int)threadIdx.x / V, vec = (int)threadIdx.x % V;
  const void* src_ptr = t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2];
  float* cent = t == 0 ? a.cent[0] : t == 1 ? a.cent[1] : a.cent[2];
  for (int x = threadIdx.x; x < 128; x += THREADS) s_tok[x] = (int)slot_token(g, j, x);
  __syncthreads();
  if (p >= map_count(a.map, g.B * g.Hd) || cent == nullptr) return;
  const int bh = map_bh(a.map, p), b = bh / g.Hd, h = bh % g.Hd;
  const uint4* src = reinterpret_cast<const uint4*>(src_ptr) + ((long long)b * g.n_tot * g.Hd + h) * V + vec;
  const long long tok_stride = (long long)g.Hd * V;   // uint4 per token
  float total[E];
#pragma unroll
  for (int e = 0; e < E; ++e) total[e] = 0.f;
#pragma unroll 1   // 64 registers: 8 CTAs per SM keep more loads in flight than a deeper unroll
  for (int r = 0; r < R; ++r) {
    uint4 x[M];
    int tok[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      tok[m] = s_tok[r + R * m];
      x[m] = tok[m] >= 0 ? __ldg(src + tok[m] * tok_stride) : make_uint4(0u, 0u, 0u, 0u);
    }
    float part[E];
#pragma unroll
    for (int e = 0; e < E; ++e) part[e] = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m)
      if (tok[m] >= 0) accumulate_vec<T>(part, x[m]);
#pragma unroll
    for (int e = 0; e < E; ++e) total[e] += part[e];
  }
  const float n = (float)block_valid_count(g, j);
  float4* out = reinterpret_cast<float4*>(cent + ((long long)bh * g.nb + j) * D + vec * E);
  out[0] = make_float4(total[0] / n, total[1] / n, total[2] / n, total[3] / n);
  out[1] = make_float4(total[4] / n, total[5] / n, total[6] / n, total[7] / n);
}

// The same pass with the optional outputs of the mask unions and the box
// estimators: (max, min) per dimension over the block's valid rows (exact in
// any order) and the SICS of SPADE §3.2 Eq. (4) as || sum_a x_a / |x_a| ||^2
// (a zero row has no direction and adds nothing).  A row's squared norm is
// summed over the V lanes that hold it (an aligned lane group of the warp);
// the unit rows are accumulated in the centroid's group order.  Threads past
// the last head still run the loop on the last head (their lanes take part
// in the shuffles) and store nothing.
template <int D>
__global__ void __launch_bounds__(kColThreads) pool_cols_extras_kernel(Geo g, GatherArgs a) {
  using T = __nv_bfloat16;
  constexpr int E = 8;                      // bf16 elements per 16-byte vector
  constexpr int V = D / E;                  // vectors per row (lanes per row)
  constexpr int R = kGatherThreads / V;     // row groups, as in gather_block
  constexpr int M = 128 / R;                // rows per group
  constexpr int HG = kColThreads / V;       // heads per CTA
  __shared__ int s_tok[128];
  const int j = blockIdx.x, t = blockIdx.z;
  const int pairs = map_count(a.map, g.B * g.Hd);
  const int p_raw = blockIdx.y * HG + (int)threadIdx.x / V, vec = (int)threadIdx.x % V;
  const bool active = p_raw < pairs;
  const int p = active ? p_raw : pairs - 1;
  const void* src_ptr = t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2];
  float* cent = t == 0 ? a.cent[0] : t == 1 ? a.cent[1] : a.cent[2];
  float* sics = t == 0 ? a.sics[0] : t == 1 ? a.sics[1] : a.sics[2];
  float* box = t == 0 ? a.box[0] : t == 1 ? a.box[1] : a.box[2];
  s_tok[threadIdx.x] = (int)slot_token(g, j, threadIdx.x);
  __syncthreads();
  const int bh = map_bh(a.map, p), b = bh / g.Hd, h = bh % g.Hd;
  const uint4* src = reinterpret_cast<const uint4*>(src_ptr) + ((long long)b * g.n_tot * g.Hd + h) * V + vec;
  const long long tok_stride = (long long)g.Hd * V;   // uint4 per token
  const bool do_sics = sics != nullptr;               // the same for the whole CTA
  float total[E], rtot[E], bmax[E], bmin[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    total[e] = rtot[e] = 0.f;
    bmax[e] = -INFINITY;
    bmin[e] = INFINITY;
  }
#pragma unroll 1
  for (int r = 0; r < R; ++r) {
    uint4 x[M];
    int tok[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      tok[m] = s_tok[r + R * m];
      x[m] = tok[m] >= 0 ? __ldg(src + tok[m] * tok_stride) : make_uint4(0u, 0u, 0u, 0u);
    }
    float part[E], rpart[E];
#pragma unroll
    for (int e = 0; e < E; ++e) part[e] = rpart[e] = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      if (tok[m] < 0) continue;   // a pad slot: the same for every thread of the CTA
      float f[E];
      to_float<T>(x[m], f);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        part[e] += f[e];
        bmax[e] = fmaxf(bmax[e], f[e]);
        bmin[e] = fminf(bmin[e], f[e]);
      }
      if (do_sics) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
        for (int o = V / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) rpart[e] = fmaf(f[e], inv, rpart[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      total[e] += part[e];
      rtot[e] += rpart[e];
    }
  }
  float sq = 0.f;
  if (do_sics) {
#pragma unroll
    for (int e = 0; e < E; ++e) sq = fmaf(rtot[e], rtot[e], sq);
#pragma unroll
    for (int o = V / 2; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  if (!active) return;
  const long long blk = (long long)bh * g.nb + j;
  if (cent != nullptr) {
    const float n = (float)block_valid_count(g, j);
    float4* out = reinterpret_cast<float4*>(cent + blk * D + vec * E);
    out[0] = make_float4(total[0] / n, total[1] / n, total[2] / n, total[3] / n);
    out[1] = make_float4(total[4] / n, total[5] / n, total[6] / n, total[7] / n);
  }
  if (box != nullptr) {
    float4* out = reinterpret_cast<float4*>(box + (blk * D + vec * E) * 2);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      out[q] = make_float4(bmax[2 * q], bmin[2 * q], bmax[2 * q + 1], bmin[2 * q + 1]);
  }
  if (do_sics && vec == 0) sics[blk] = sq;
}

// Aggregation evaluation (SPADE §3.2): SICS of every block of every candidate
// blocking scheme, read from the original layout.  One warp per (b, h,
// candidate, block): the online form of Eq. (5), a running sum of unit rows
// per lane, with no block barrier.  A lane holds kSicsChunks 16-byte pieces of
// a row, so L lanes share one row of D elements and one warp step covers
// RPI = 32 / L rows; piece k of lane v is row bytes [(k L + v) 16, +16), so
// every copy instruction reads whole 128-byte segments.  Each warp streams its
// rows through a private kSicsStages-deep shared-memory ring with 16-byte
// cp.async copies (rows past the block's end are zero-filled, not read), so
// that kSicsStages steps per warp are in flight without holding registers.
// Warps are numbered head-major, then candidate, then block: the candidates
// of one head run back to back and re-read its rows from L2 (HBM traffic is
// one read of x whatever the number of candidates).
constexpr int kSicsWarps = 4;
constexpr int kSicsStages = 4;
constexpr int kSicsChunks = 4;


template <typename T, int D>
__global__ void __launch_bounds__(kSicsWarps * 32, 4) sics_schemes_kernel(SchemeArgs s, int per_bh,
                                                                        long long n_tasks) {
  constexpr int E = 16 / (int)sizeof(T);          // elements per 16-byte piece
  constexpr int C = kSicsChunks;
  constexpr int L = D / (E * C);                  // lanes per row
  constexpr int RPI = 32 / L;                     // rows per warp step
  static_assert(L >= 1 && L <= 32 && 32 % L == 0, "row split");
  __shared__ __align__(16) uint4 s_ring[kSicsWarps][kSicsStages][C][32];
  const int warp = threadIdx.x >> 5;
  const long long task = (long long)blockIdx.x * kSicsWarps + warp;
  if (task >= n_tasks) return;
  const int lane = threadIdx.x & 31, sub = lane / L, vec = lane % L;
  const int bh = (int)(task / per_bh);
  int j = (int)(task % per_bh), c = 0;
  while (j >= s.g[c].nb) j -= s.g[c++].nb;
  const Geo& g = s.g[c];
  const int b = bh / g.Hd, h = bh % g.Hd;
  const int xb = j % g.nbx, yb = (j / g.nbx) % g.nby, tb = j / (g.nbx * g.nby);
  const int t0 = tb * g.bf, y0 = yb * g.br, x0 = xb * g.bc;
  const int vt = min(g.bf, g.T - t0), vy = min(g.br, g.H - y0), vx = min(g.bc, g.W - x0);
  const int n = vt * vy * vx;
  const int n_steps = (n + RPI - 1) / RPI;
  // (dt, dy, dx) of this lane's next row (row `sub`, then +RPI per step) and
  // the row's address, advanced with carries instead of divisions.
  const long long sx = (long long)g.Hd * L * C;          // 16-byte pieces per token
  const long long sy = sx * g.W, st = sy * g.H;
  const uint4* first = reinterpret_cast<const uint4*>(s.x) +
                       ((long long)b * g.n_tot * g.Hd + h) * (L * C) + vec +
                       ((long long)t0 * g.H + y0) * sy + (long long)x0 * sx;
  const uint4* ptr = first;
  int dx = 0, dy = 0, dt = 0;
  auto advance = [&](int k) {
    dx += k;
    ptr += k * sx;
    while (dx >= vx && dt < vt) {
      dx -= vx;
      ptr += sy - vx * sx;
      if (++dy >= vy) {
        dy = 0;
        ++dt;
        ptr += st - vy * sy;
      }
    }
  };
  advance(sub);
  const uint32_t ring = smem_addr(&s_ring[warp][0][0][lane]);
  auto issue = [&](int step) {   // steps are issued in order 0, 1, 2, ...
    const bool ok = step * RPI + sub < n;
    const uint32_t dst = ring + (uint32_t)((step % kSicsStages) * C * 32 * 16);
#pragma unroll
    for (int k = 0; k < C; ++k)
      cp_async16(dst + k * 32 * 16, ok ? ptr + k * L : first, ok ? 16u : 0u);
    advance(RPI);
  };
#pragma unroll
  for (int k = 0; k < kSicsStages - 1; ++k) {
    if (k < n_steps) issue(k);
    cp_async_commit();
  }
  float2 racc[C * E / 2];
#pragma unroll
  for (int e = 0; e < C * E / 2; ++e) racc[e] = make_float2(0.f, 0.f);
  for (int i = 0; i < n_steps; ++i) {
    if (i + kSicsStages - 1 < n_steps) issue(i + kSicsStages - 1);
    cp_async_commit();
    cp_async_wait<kSicsStages - 1>();   // this lane's copies of step i have landed
    float2 f[C * E / 2];
#pragma unroll
    for (int k = 0; k < C; ++k) to_float<T>(s_ring[warp][i % kSicsStages][k][lane],
                                            reinterpret_cast<float*>(f + k * E / 2));
    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < C * E / 2; ++e) ss2 = fma2(f[e], f[e], ss2);
    float ss = ss2.x + ss2.y;
#pragma unroll
    for (int o = L / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int e = 0; e < C * E / 2; ++e) racc[e] = fma2(f[e], inv2, racc[e]);
  }
  cp_async_wait<0>();
  // r = sum over the RPI row groups; |r|^2 = sum over the L lanes of one group
  float r2 = 0.f;
#pragma unroll
  for (int e = 0; e < C * E / 2; ++e) {
    float rx = racc[e].x, ry = racc[e].y;
#pragma unroll
    for (int o = L; o < 32; o <<= 1) {
      rx += __shfl_xor_sync(0xffffffffu, rx, o);
      ry += __shfl_xor_sync(0xffffffffu, ry, o);
    }
    r2 = fmaf(rx, rx, r2);
    r2 = fmaf(ry, ry, r2);
  }
#pragma unroll
  for (int o = L / 2; o >= 1; o >>= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, o);
  if (lane == 0) s.sics[c][(long long)bh * g.nb + j] = r2;
}

// Aggregation score AS(x | scheme c) = sum over the video blocks of SICS
// (SPADE §3.2, Eq. (3)), summed in double in a fixed order, and the
// per-(b, h) choice of the scheme with the largest AS (lowest candidate
// index among equal scores).  One warp per (b, h).
__global__ void __launch_bounds__(128) aggregate_kernel(SchemeArgs s, int BH) {
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (bh >= BH) return;
  double best = 0.0;
  int arg = 0;
  for (int c = 0; c < s.n; ++c) {
    const int nb = s.g[c].nb;
    const float* src = s.sics[c] + (long long)bh * nb;
    double t = 0.0;
    for (int jj = lane; jj < nb; jj += 32) t += (double)src[jj];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (s.as != nullptr && lane == 0) s.as[(long long)c * BH + bh] = t;
    if (c == 0 || t > best) {
      best = t;
      arg = c;
    }
  }
  if (s.choice != nullptr && lane == 0) s.choice[bh] = arg;
}

template <typename T, int MODE>
static cudaError_t launch_gather_t(const Geo& g, const GatherArgs& a, int nblocks,
                                   cudaStream_t st) {
  dim3 grid(nblocks, a.map.n ? a.map.n : g.Hd, a.map.n ? a.ntensors : g.B * a.ntensors);
  bool extras = false;
  for (int t = 0; t < a.ntensors; ++t) extras = extras || a.sics[t] != nullptr || a.box[t] != nullptr;
  if (MODE != kUnpermute && extras) {
    if (g.D == 128)
      gather_kernel<T, 128, MODE, true><<<grid, kGatherThreads, 0, st>>>(g, a);
    else
      gather_kernel<T, 64, MODE, true><<<grid, kGatherThreads, 0, st>>>(g, a);
  } else {
    if (g.D == 128)
      gather_kernel<T, 128, MODE, false><<<grid, kGatherThreads, 0, st>>>(g, a);
    else
      gather_kernel<T, 64, MODE, false><<<grid, kGatherThreads, 0, st>>>(g, a);
  }
  return cudaGetLastError();
}

// Launchers.  is_bf16 selects the element type; D must be 64 or 128.
cudaError_t launch_permute(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  const int nblocks = g.nb + g.nb_text;
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kPermute>(g, a, nblocks, st)
                 : launch_gather_t<float, kPermute>(g, a, nblocks, st);
}

cudaError_t launch_unpermute(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  const int nblocks = g.nb + g.nb_text;
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kUnpermute>(g, a, nblocks, st)
                 : launch_gather_t<float, kUnpermute>(g, a, nblocks, st);
}

// Multiprocessors of the current device (queried once per device).
static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cached[dev] = (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
                      ? n : 148;
  }
  return cached[dev];
}

// Centroids of the video blocks straight from the original layout (the
// summarizer pass of the fused forward, which never materialises the blocked
// tensors).
cudaError_t launch_pool_orig(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  bool extras = false;
  for (int t = 0; t < a.ntensors; ++t) extras = extras || a.sics[t] != nullptr || a.box[t] != nullptr;
  if (is_bf16 && g.bs == 128 && (g.D == 128 || g.D == 64)) {
    const int pairs = map_count(a.map, g.B * g.Hd);
    const int hg = kColThreads / (g.D / 8);
    const dim3 grid(g.nb, (pairs + hg - 1) / hg, a.ntensors);
    if (g.nb == 0 || pairs == 0) return cudaSuccess;
    if (extras) {
      if (g.D == 128) pool_cols_extras_kernel<128><<<grid, kColThreads, 0, st>>>(g, a);
      else pool_cols_extras_kernel<64><<<grid, kColThreads, 0, st>>>(g, a);
      return cudaGetLastError();
    }
    // Heads per CTA: 128 threads (8 CTAs per SM at 64 registers a thread,
    // the most loads in flight) unless 192 or 256 threads (5 or 4 CTAs per
    // SM) need fewer waves of CTA slots.  Wan2.1-1.3B's 12 heads: 192
    // threads, one head group, 672 CTAs in one wave of 740 slots instead of
    // 1344 in 1184 (centroids 43 -> 37 us); HunyuanVideo, Wan2.1-14B and
    // Long keep 128 (as many waves either way; 192 measured slower there).
    const int V = g.D / 8;
    const int sms = sm_count();
    auto waves = [&](int threads) {
      const int hgc = threads / V;
      const long long ctas = (long long)g.nb * ((pairs + hgc - 1) / hgc) * a.ntensors;
      const long long slots = (long long)sms * (65536 / (threads * 64));
      return (ctas + slots - 1) / slots;
    };
    int best = 128;
    for (int threads : {192, 256})
      if (waves(threads) < waves(best)) best = threads;
    const dim3 grid_b(g.nb, (pairs + best / V - 1) / (best / V), a.ntensors);
    if (g.D == 128) {
      if (best == 192) pool_cols_kernel<128, 192><<<grid_b, 192, 0, st>>>(g, a);
      else if (best == 256) pool_cols_kernel<128, 256><<<grid_b, 256, 0, st>>>(g, a);
      else pool_cols_kernel<128, 128><<<grid_b, 128, 0, st>>>(g, a);
    } else {
      if (best == 192) pool_cols_kernel<64, 192><<<grid_b, 192, 0, st>>>(g, a);
      else if (best == 256) pool_cols_kernel<64, 256><<<grid_b, 256, 0, st>>>(g, a);
      else pool_cols_kernel<64, 128><<<grid_b, 128, 0, st>>>(g, a);
    }
    return cudaGetLastError();
  }
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kPoolOrig>(g, a, g.nb, st)
                 : launch_gather_t<float, kPoolOrig>(g, a, g.nb, st);
}

// Centroids of the video blocks straight from the blocked layout.
cudaError_t launch_pool(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kPool>(g, a, g.nb, st)
                 : launch_gather_t<float, kPool>(g, a, g.nb, st);
}

cudaError_t launch_sics_schemes(const SchemeArgs& a, bool is_bf16, cudaStream_t st) {
  const Geo& g0 = a.g[0];
  int per_bh = 0;
  for (int c = 0; c < a.n; ++c) per_bh += a.g[c].nb;
  const int BH = g0.B * g0.Hd;
  const long long n_tasks = (long long)per_bh * BH;
  if (n_tasks > 0) {
    const long long grid = (n_tasks + kSicsWarps - 1) / kSicsWarps;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const dim3 gd((unsigned)grid), bd(kSicsWarps * 32);
    if (is_bf16) {
      if (g0.D == 128) sics_schemes_kernel<__nv_bfloat16, 128><<<gd, bd, 0, st>>>(a, per_bh, n_tasks);
      else sics_schemes_kernel<__nv_bfloat16, 64><<<gd, bd, 0, st>>>(a, per_bh, n_tasks);
    } else {
      if (g0.D == 128) sics_schemes_kernel<float, 128><<<gd, bd, 0, st>>>(a, per_bh, n_tasks);
      else sics_schemes_kernel<float, 64><<<gd, bd, 0, st>>>(a, per_bh, n_tasks);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.as != nullptr || a.choice != nullptr)
    aggregate_kernel<<<(BH + 3) / 4, 128, 0, st>>>(a, BH);
  return cudaGetLastError();
}

}  // namespace bsa
