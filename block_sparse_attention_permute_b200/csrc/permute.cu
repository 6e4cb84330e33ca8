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

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(Geo g, GatherArgs a) {
  constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte vector
  constexpr int V = D / E;                // vectors per row
  constexpr int R = kGatherThreads / V;   // rows per pass
  __shared__ int s_tok[256];
  __shared__ float s_red[R * D];

  const int j = blockIdx.x, h = blockIdx.y;
  const int tensor = blockIdx.z % a.ntensors, b = blockIdx.z / a.ntensors;
  const int tid = threadIdx.x, row0 = tid / V, vec = tid % V;

  for (int s = tid; s < g.bs; s += kGatherThreads) s_tok[s] = (int)slot_token(g, j, s);
  __syncthreads();

  const long long blk_row0 = (long long)(b * g.Hd + h) * g.npad_tot + (long long)j * g.bs;
  const long long tok_base = (long long)b * g.n_tot;
  float* cent = (MODE != kUnpermute && j < g.nb) ? a.cent[tensor] : nullptr;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;

  const uint4* src = reinterpret_cast<const uint4*>(a.src[tensor]);
  uint4* dst = reinterpret_cast<uint4*>(a.dst[tensor]);
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
}

template <typename T, int MODE>
static cudaError_t launch_gather_t(const Geo& g, const GatherArgs& a, int nblocks,
                                   cudaStream_t st) {
  dim3 grid(nblocks, g.Hd, g.B * a.ntensors);
  if (g.D == 128)
    gather_kernel<T, 128, MODE><<<grid, kGatherThreads, 0, st>>>(g, a);
  else
    gather_kernel<T, 64, MODE><<<grid, kGatherThreads, 0, st>>>(g, a);
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

// Centroids of the video blocks straight from the original layout (the
// summarizer pass of the fused forward, which never materialises the blocked
// tensors).
cudaError_t launch_pool_orig(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kPoolOrig>(g, a, g.nb, st)
                 : launch_gather_t<float, kPoolOrig>(g, a, g.nb, st);
}

// Centroids of the video blocks straight from the blocked layout.
cudaError_t launch_pool(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st) {
  return is_bf16 ? launch_gather_t<__nv_bfloat16, kPool>(g, a, g.nb, st)
                 : launch_gather_t<float, kPool>(g, a, g.nb, st);
}

}  // namespace bsa
