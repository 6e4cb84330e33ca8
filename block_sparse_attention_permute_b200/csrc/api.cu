// api.cu — the C ABI of libbsa (declared in include/bsa.h): argument
// validation, plan state, workspace carving, TMA tensor maps and launches.
// Every entry point validates on the host before it launches anything.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "bsa.h"
#include "kernels.cuh"

struct bsa_plan_s {
  Geo g;
  bsa_dtype dtype;
  int device;
  int attn_path;        // 1 tcgen05, 0 SIMT
  int32_t* d_status;    // device status word
  long long wait_limit; // bound of the attention kernel's waits, SM cycles (0 = default)
  int hold_load;        // test hook of the timeout path (0 = off)
  uint32_t* d_masks;    // [(nb + nb_text) * 4] slot validity bits (bs == 128)
};

namespace {

thread_local std::string g_err;

bsa_status fail(bsa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

bsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

size_t elem_size(const bsa_plan_s* p) { return p->dtype == BSA_BF16 ? 2 : 4; }

size_t blk_bytes(const bsa_plan_s* p) {
  return (size_t)p->g.B * p->g.Hd * p->g.npad_tot * p->g.D * elem_size(p);
}
size_t cent_bytes(const bsa_plan_s* p) {
  return (size_t)p->g.B * p->g.Hd * p->g.nb * p->g.D * sizeof(float);
}

// k per head for a density (the fraction of key blocks each query block keeps).
int k_for_density(double rho, int nb) {
  long long k = (long long)std::ceil(rho * (double)nb - 1e-9);
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return (int)k;
}

bsa_status check_params(const bsa_plan_s* p, bsa_select_mode mode, const double* param,
                        int* kmax_needed) {
  if (param == nullptr) return fail(BSA_ERR_INVALID_ARG, "param_per_head is NULL");
  if (mode != BSA_TOPK && mode != BSA_TOPP) return fail(BSA_ERR_INVALID_ARG, "bad select mode %d", (int)mode);
  int kmax = 0;
  for (int h = 0; h < p->g.Hd; ++h) {
    const double v = param[h];
    if (!(v > 0.0 && v <= 1.0))
      return fail(BSA_ERR_INVALID_ARG, "%s of head %d is %g, must be in (0, 1]",
                  mode == BSA_TOPK ? "density" : "tau", h, v);
    const int k = mode == BSA_TOPK ? k_for_density(v, p->g.nb) : p->g.nb;
    if (k > kmax) kmax = k;
  }
  *kmax_needed = kmax + p->g.nb_text;
  return BSA_OK;
}

bsa_status check_plan(const bsa_plan_s* p) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "plan is NULL");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != p->device)
    return fail(BSA_ERR_INVALID_ARG, "plan was created on device %d, current device is %d", p->device, dev);
  return BSA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D map over a blocked bf16 tensor: rows x D, box 64 x 128, 128-byte swizzle.
bsa_status make_tile_map(CUtensorMap* m, const void* base, long long rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return BSA_OK;
}

CUresult encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box) {
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                     dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Maps over ONE batch element of an original-layout tensor [Ntot, Hd, D]:
// video tokens as a 5D tensor (d, head, x, y, t) with box (64, 1, bc, br, bf)
// (rows land in slot order, the padded part of the box reads zeros); text
// tokens as a 3D tensor (d, head, token) with box (64, 1, 128).
bsa_status make_orig_maps(CUtensorMap* video, CUtensorMap* text, const void* x, const Geo& g) {
  if (encode_fn() == nullptr) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t row = (cuuint64_t)g.D * 2;                    // bytes per (token, head) row
  const cuuint64_t tok = row * g.Hd;                             // bytes per token
  cuuint64_t vd[5] = {(cuuint64_t)g.D, (cuuint64_t)g.Hd, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
  cuuint64_t vs[4] = {row, tok, tok * g.W, tok * g.W * g.H};
  cuuint32_t vb[5] = {64, 1, (cuuint32_t)g.bc, (cuuint32_t)g.br, (cuuint32_t)g.bf};
  CUresult r = encode(video, x, 5, vd, vs, vb);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (video) failed (%d)", (int)r);
  std::memset(text, 0, sizeof(*text));
  if (g.n_text > 0) {
    const char* tbase = reinterpret_cast<const char*>(x) + tok * g.n_video;
    cuuint64_t td[3] = {(cuuint64_t)g.D, (cuuint64_t)g.Hd, (cuuint64_t)g.n_text};
    cuuint64_t ts[2] = {row, tok};
    cuuint32_t tb[3] = {64, 1, 128};
    r = encode(text, tbase, 3, td, ts, tb);
    if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (text) failed (%d)", (int)r);
  }
  return BSA_OK;
}

// Events at the phase boundaries of one forward call (bsa_forward_timed):
// mark() records the next event on the call's stream; a null timer records
// nothing.
struct PhaseTimer {
  cudaEvent_t ev[6];
  int n = 0;
  cudaStream_t st = nullptr;
  cudaError_t err = cudaSuccess;
};
void mark(PhaseTimer* t) {
  if (t == nullptr || t->n >= 6 || t->err != cudaSuccess) return;
  t->err = cudaEventRecord(t->ev[t->n++], t->st);
}

// Host copy of a validated mask union (window, sink, intra selection).
struct UnionOpts {
  int win_left = -1, win_right = -1;
  long long sink_tokens = 0;
  bool intra = false;
  int intra_mode = 0;
  double intra_param[BSA_MAX_HEADS] = {};   // k (held in a double) or tau per head; <= 0 = none
};

size_t bits_bytes(const bsa_plan_s* p) {
  return (size_t)p->g.B * p->g.Hd * ((p->g.nb + 31) / 32) * sizeof(uint32_t);
}
size_t sics_bytes(const bsa_plan_s* p) { return (size_t)p->g.B * p->g.Hd * p->g.nb * sizeof(float); }

// Validates `u` (NULL = no union) and returns the number of video key blocks
// it can add to one list on top of the inter selection.
bsa_status check_union(const bsa_plan_s* p, const bsa_mask_union_t* u, UnionOpts* o, int* extra) {
  *o = UnionOpts();
  *extra = 0;
  if (u == nullptr) return BSA_OK;
  const int nb = p->g.nb;
  o->win_left = u->window_left;
  o->win_right = u->window_right;
  o->sink_tokens = u->sink_tokens;
  if (u->sink_tokens < 0) return fail(BSA_ERR_INVALID_ARG, "sink_tokens must be >= 0");
  long long add = 0;
  if (u->window_left >= 0 || u->window_right >= 0)
    add += (u->window_left < 0 || u->window_right < 0)
               ? nb : (long long)u->window_left + u->window_right + 1;
  if (u->sink_tokens > 0) {
    const Geo& g = p->g;
    for (int j = 0; j < nb; ++j) {
      const int xb = j % g.nbx, yb = (j / g.nbx) % g.nby, tb = j / (g.nbx * g.nby);
      const long long first = ((long long)tb * g.bf * g.H + (long long)yb * g.br) * g.W +
                              (long long)xb * g.bc;
      if (first < u->sink_tokens) ++add;
    }
  }
  if (u->intra_param != nullptr) {
    if (u->intra_mode != BSA_TOPK && u->intra_mode != BSA_TOPP)
      return fail(BSA_ERR_INVALID_ARG, "bad intra mode %d", (int)u->intra_mode);
    o->intra_mode = (int)u->intra_mode;
    int kmax_intra = 0;
    for (int h = 0; h < p->g.Hd; ++h) {
      const double v = u->intra_param[h];
      if (!(v >= 0.0 && v <= 1.0))
        return fail(BSA_ERR_INVALID_ARG, "intra %s of head %d is %g, must be in [0, 1]",
                    u->intra_mode == BSA_TOPK ? "density" : "tau", h, v);
      if (v > 0.0) {
        o->intra = true;
        o->intra_param[h] = u->intra_mode == BSA_TOPK ? (double)k_for_density(v, nb) : v;
        const int k = u->intra_mode == BSA_TOPK ? k_for_density(v, nb) : nb;
        if (k > kmax_intra) kmax_intra = k;
      }
    }
    add += kmax_intra;
  }
  *extra = (int)(add < nb ? add : nb);
  return BSA_OK;
}

bsa_status run_select(const bsa_plan_s* p, const float* qc, const float* kc, bsa_select_mode mode,
                      const double* param, int kmax, int32_t* idx, int32_t* cnt, float* scores,
                      cudaStream_t st, const UnionOpts* uo = nullptr, const float* intra_scores = nullptr,
                      uint32_t* bits = nullptr, int est = bsa::kEstMean,
                      const bsa::HeadMap* map = nullptr, uint32_t* list_bits = nullptr) {
  int need = 0;
  bsa_status s = check_params(p, mode, param, &need);
  if (s != BSA_OK) return s;
  // (union callers check kmax against the union's bound themselves)
  if (kmax < need) return fail(BSA_ERR_INVALID_ARG, "kmax %d is below the %d entries a list can need", kmax, need);
  if (p->g.nb == 0) return BSA_OK;
  if (!qc || !kc || !idx || !cnt) return fail(BSA_ERR_INVALID_ARG, "NULL centroid or list pointer");
  if (!aligned16(qc) || !aligned16(kc)) return fail(BSA_ERR_INVALID_ARG, "summaries must be 16-byte aligned");
  if (est != bsa::kEstMean && bsa::select_smem_bytes(p->g.nb, 2 * p->g.D, 8) > 227 * 1024)
    return fail(BSA_ERR_UNSUPPORTED, "nb = %d is too large for the box estimators", p->g.nb);
  bsa::SelectArgs a;
  std::memset(&a, 0, sizeof(a));
  a.qc = qc; a.kc = kc; a.idx = idx; a.cnt = cnt; a.scores = scores; a.kmax = kmax;
  a.list_bits = list_bits;
  a.mode = (int)mode;
  a.est = est;
  if (map) a.map = *map;
  a.scale = (float)(1.0 / std::sqrt((double)p->g.D));
  for (int h = 0; h < p->g.Hd; ++h)
    a.param[h] = mode == BSA_TOPK ? (double)k_for_density(param[h], p->g.nb) : param[h];
  a.win_left = a.win_right = -1;
  if (uo != nullptr) {
    a.win_left = uo->win_left;
    a.win_right = uo->win_right;
    a.sink_tokens = uo->sink_tokens;
    if (uo->intra) {
      if (!intra_scores || !bits) return fail(BSA_ERR_INVALID_ARG, "intra selection needs intra scores");
      bsa::IntraArgs ia;
      std::memset(&ia, 0, sizeof(ia));
      ia.scores = intra_scores;
      ia.bits = bits;
      ia.mode = uo->intra_mode;
      if (map) ia.map = *map;
      for (int h = 0; h < p->g.Hd; ++h) ia.param[h] = uo->intra_param[h];
      cudaError_t e = bsa::launch_intra_select(p->g, ia, st);
      if (e != cudaSuccess) return cuda_fail(e, "intra select kernel");
      a.intra_bits = bits;
    }
  }
  cudaError_t e = bsa::launch_select(p->g, a, st);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "select kernel");
}

bsa_status run_attention(const bsa_plan_s* p, const void* q, const void* k, const void* v,
                         const int32_t* idx, const int32_t* cnt, int kmax, void* o,
                         int32_t* dev_status, cudaStream_t st) {
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_INVALID_ARG, "blocked tensors must be 16-byte aligned");
  if (p->g.nb > 0 && (!idx || !cnt)) return fail(BSA_ERR_INVALID_ARG, "NULL index list");
  if (kmax < 1) return fail(BSA_ERR_INVALID_ARG, "kmax must be >= 1");
  bsa::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.o = o; a.idx = idx; a.cnt = cnt; a.masks = p->d_masks;
  a.status = dev_status ? dev_status : p->d_status;
  a.kmax = kmax;
  a.wait_limit = p->wait_limit;
  a.hold_load = p->hold_load;
  a.div_nbx = make_fastdiv((uint32_t)p->g.nbx);
  a.div_nby = make_fastdiv((uint32_t)p->g.nby);
  a.div_hd = make_fastdiv((uint32_t)p->g.Hd);
  a.scale = (float)(1.0 / std::sqrt((double)p->g.D));
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->g.D));
  cudaError_t e;
  if (p->attn_path == 1) {
    bsa::TileMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const long long rows = (long long)p->g.B * p->g.Hd * p->g.npad_tot;
    bsa_status s;
    if ((s = make_tile_map(&maps.q, q, rows, p->g.D)) != BSA_OK) return s;
    if ((s = make_tile_map(&maps.k, k, rows, p->g.D)) != BSA_OK) return s;
    if ((s = make_tile_map(&maps.v, v, rows, p->g.D)) != BSA_OK) return s;
    e = bsa::launch_attn_tc(p->g, a, maps, st);
  } else {
    e = bsa::launch_attn_simt(p->g, p->dtype == BSA_BF16, a, st);
  }
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "attention kernel");
}

// Summaries straight from the original layout: centroids (MEAN) or (max,
// min) boxes (DSA, DSA2) of Q and K, optionally with the SICS of the K blocks.
bsa_status run_centroids(const bsa_plan_s* p, const void* q, const void* k, float* qc, float* kc,
                         cudaStream_t st, float* k_sics = nullptr, bool boxes = false,
                         const bsa::HeadMap* map = nullptr) {
  // Only the requested tensors are read.
  bsa::GatherArgs ga;
  std::memset(&ga, 0, sizeof(ga));
  if (map) ga.map = *map;
  if (qc) {
    ga.src[ga.ntensors] = q;
    (boxes ? ga.box : ga.cent)[ga.ntensors] = qc;
    ++ga.ntensors;
  }
  if (kc) {
    ga.src[ga.ntensors] = k;
    (boxes ? ga.box : ga.cent)[ga.ntensors] = kc;
    ga.sics[ga.ntensors] = k_sics;
    ++ga.ntensors;
  }
  if (ga.ntensors == 0 || p->g.nb == 0) return BSA_OK;
  cudaError_t e = bsa::launch_pool_orig(p->g, p->dtype == BSA_BF16, ga, st);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "centroid kernel");
}

// Attention on the original layout, one launch per batch element.
// Query tiles per head paired for K/V sharing (pair.cu): text pairs, then
// video pairs.
int text_pairs(const Geo& g) { return (g.nb_text + 1) / 2; }
// Text pairs of the paired schedule run as key chunks of about two lists
// (each about as long as two video pairs, read within its head's window);
// their partial rows are merged afterwards.  Measured on HunyuanVideo: one
// list per chunk and two lists per chunk cut the attention's DRAM reads the
// same (2.14 -> 1.33 GB), two costing less time (fewer CTA prologues).
int text_chunk_len(const Geo& g, int kmax) {
  const int nbk = g.nb + g.nb_text;
  return std::min(nbk, std::max(32, 2 * kmax));
}
int text_chunks(const Geo& g, int kmax) {
  const int len = text_chunk_len(g, kmax);
  return (g.nb + g.nb_text + len - 1) / len;
}
// Partial rows of the text chunks of one batch element (reused per element).
size_t text_part_bytes(const Geo& g, int kmax) {
  return (size_t)g.Hd * g.nb_text * text_chunks(g, kmax) * 128 * (g.D + 4) * sizeof(float);
}
int pairs_per_head(const Geo& g) { return text_pairs(g) + (g.nb + 1) / 2; }
size_t pairing_bytes(const bsa_plan_s* p, int kmax) {
  const size_t bh = (size_t)p->g.B * p->g.Hd, pph = pairs_per_head(p->g);
  return round256(bsa::pair_scratch_bytes(p->g)) + round256(bh * pph * 4 * sizeof(int32_t)) +
         round256(bh * pph * 2 * (size_t)kmax * sizeof(int32_t)) + round256(text_part_bytes(p->g, kmax));
}
// The text partials' place in a pairing workspace (after the lists).
float* text_part_of(const bsa_plan_s* p, int kmax, char* w) {
  const size_t bh = (size_t)p->g.B * p->g.Hd, pph = pairs_per_head(p->g);
  return reinterpret_cast<float*>(w + round256(bsa::pair_scratch_bytes(p->g)) +
                                  round256(bh * pph * 4 * sizeof(int32_t)) +
                                  round256(bh * pph * 2 * (size_t)kmax * sizeof(int32_t)));
}

// Pairs the query tiles of the selected heads (scratch and schedule carved
// from `w`, pairing_bytes long); on return *sched / *lists point at them.
// With bits_ready the lists' bit sets are already at the start of `w`
// (written by the selection).
bsa_status run_pairing(const bsa_plan_s* p, const int32_t* idx, const int32_t* cnt, int kmax,
                       char* w, int32_t** sched, int32_t** lists, cudaStream_t st,
                       const bsa::HeadMap* map, bool bits_ready = false) {
  const size_t bh = (size_t)p->g.B * p->g.Hd, pph = pairs_per_head(p->g);
  const size_t nbw = (p->g.nb + 31) / 32;
  bsa::PairArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  pa.idx = idx;
  pa.cnt = cnt;
  pa.bits = reinterpret_cast<uint32_t*>(w);
  pa.cand = reinterpret_cast<uint16_t*>(w + round256(bh * p->g.nb * nbw * sizeof(uint32_t)));
  w += round256(bsa::pair_scratch_bytes(p->g));
  pa.sched = reinterpret_cast<int32_t*>(w);
  w += round256(bh * pph * 4 * sizeof(int32_t));
  pa.lists = reinterpret_cast<int32_t*>(w);
  pa.kmax = kmax;
  pa.pairs_per_head = (int)pph;
  pa.text_pairs = text_pairs(p->g);
  pa.bits_ready = bits_ready ? 1 : 0;
  if (map) pa.map = *map;
  cudaError_t e = bsa::launch_pairing(p->g, pa, st);
  if (e != cudaSuccess) return cuda_fail(e, "pairing kernels");
  *sched = pa.sched;
  *lists = pa.lists;
  return BSA_OK;
}

bsa_status run_attention_orig(const bsa_plan_s* p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const int32_t* cnt, int kmax, void* o,
                              int32_t* dev_status, cudaStream_t st,
                              const bsa::HeadMap* map = nullptr,
                              const int32_t* pair_sched = nullptr,
                              const int32_t* pair_lists = nullptr, float* part = nullptr) {
  if (p->attn_path != 1)
    return fail(BSA_ERR_UNSUPPORTED, "attention on the original layout needs a bf16 plan with 128-token blocks");
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (p->g.nb > 0 && (!idx || !cnt)) return fail(BSA_ERR_INVALID_ARG, "NULL index list");
  if (kmax < 1) return fail(BSA_ERR_INVALID_ARG, "kmax must be >= 1");
  const size_t per_batch = (size_t)p->g.n_tot * p->g.Hd * p->g.D * 2;
  Geo g1 = p->g;
  g1.B = 1;
  bsa_status s;
  for (int b = 0; b < p->g.B; ++b) {
    // the heads of this batch element that the map selects (all without one)
    bsa::HeadMap hm;
    std::memset(&hm, 0, sizeof(hm));
    if (map && map->n) {
      for (int x = 0; x < map->n; ++x)
        if (map->bh[x] / p->g.Hd == b) hm.bh[hm.n++] = (uint8_t)(map->bh[x] % p->g.Hd);
      if (hm.n == 0) continue;
    }
    bsa::TileMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const char* qb = reinterpret_cast<const char*>(q) + b * per_batch;
    const char* kb = reinterpret_cast<const char*>(k) + b * per_batch;
    const char* vb = reinterpret_cast<const char*>(v) + b * per_batch;
    if ((s = make_orig_maps(&maps.q, &maps.qt, qb, p->g)) != BSA_OK) return s;
    if ((s = make_orig_maps(&maps.k, &maps.kt, kb, p->g)) != BSA_OK) return s;
    if ((s = make_orig_maps(&maps.v, &maps.vt, vb, p->g)) != BSA_OK) return s;
    bsa::AttnArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = qb; a.k = kb; a.v = vb;
    a.o = reinterpret_cast<char*>(o) + b * per_batch;
    a.idx = idx + (size_t)b * p->g.Hd * p->g.nb * kmax;
    a.cnt = cnt + (size_t)b * p->g.Hd * p->g.nb;
    a.masks = p->d_masks;
    a.status = dev_status ? dev_status : p->d_status;
    a.kmax = kmax;
    a.wait_limit = p->wait_limit;
    a.hold_load = p->hold_load;
    a.div_nbx = make_fastdiv((uint32_t)p->g.nbx);
    a.div_nby = make_fastdiv((uint32_t)p->g.nby);
    a.div_hd = make_fastdiv((uint32_t)p->g.Hd);
    a.scale = (float)(1.0 / std::sqrt((double)p->g.D));
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->g.D));
    a.map = hm;
    if (pair_sched != nullptr) {
      const long long pph = pairs_per_head(p->g);
      a.pair_sched = pair_sched + (long long)b * p->g.Hd * pph * 4;
      a.pair_lists = pair_lists + (long long)b * p->g.Hd * pph * 2 * kmax;
      a.pairs_per_head = (int)pph;
      a.text_pairs = text_pairs(p->g);
      a.text_chunk_len = text_chunk_len(p->g, kmax);
      a.text_chunks = text_chunks(p->g, kmax);
      a.part = part;
    }
    cudaError_t e = bsa::launch_attn_tc_orig(g1, a, maps, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
    if (pair_sched != nullptr && p->g.nb_text > 0) {
      bsa::MergeArgs ma;
      std::memset(&ma, 0, sizeof(ma));
      ma.part = part;
      ma.o = a.o;
      ma.text_chunks = a.text_chunks;
      ma.map = hm;
      if ((e = bsa::launch_text_merge(g1, ma, st)) != cudaSuccess) return cuda_fail(e, "text merge kernel");
    }
  }
  return BSA_OK;
}

// The fused forward of the tensor-core path: centroids from the original
// layout, selection, then attention that gathers its tiles from the original
// layout and scatters the output back.
bsa_status run_forward_fused(const bsa_plan_s* p, const void* q, const void* k, const void* v,
                             bsa_select_mode mode, const double* param, int kmax, void* o,
                             int32_t* idx, int32_t* cnt, float* qc, float* kc,
                             int32_t* dev_status, cudaStream_t st, const UnionOpts* uo,
                             float* k_sics, uint32_t* bits, int est, char* pair_ws,
                             const bsa::HeadMap* map = nullptr, PhaseTimer* timer = nullptr) {
  mark(timer);
  bsa_status s = run_centroids(p, q, k, qc, kc, st, k_sics, est != bsa::kEstMean, map);
  if (s != BSA_OK) return s;
  mark(timer);
  // pairing only reorders the work; plans beyond its block limit run unpaired
  const bool paired = pair_ws != nullptr && bsa::pairing_supported(p->g);
  // the selection writes the lists' bit sets straight into the pairing scratch
  uint32_t* list_bits = paired ? reinterpret_cast<uint32_t*>(pair_ws) : nullptr;
  if ((s = run_select(p, qc, kc, mode, param, kmax, idx, cnt, nullptr, st, uo, k_sics, bits, est,
                      map, list_bits)) != BSA_OK)
    return s;
  mark(timer);
  int32_t* sched = nullptr;
  int32_t* lists = nullptr;
  if (paired && (s = run_pairing(p, idx, cnt, kmax, pair_ws, &sched, &lists, st, map, true)) != BSA_OK)
    return s;
  mark(timer);
  s = run_attention_orig(p, q, k, v, idx, cnt, kmax, o, dev_status, st, map, sched, lists,
                         sched ? text_part_of(p, kmax, pair_ws) : nullptr);
  mark(timer);
  return s;
}

// kmax a list can need under the union: the inter bound plus the blocks the
// union can add, at most every video block, plus the text blocks.
bsa_status union_kmax(const bsa_plan_s* p, bsa_select_mode mode, const double* param,
                      const bsa_mask_union_t* u, int* kmax) {
  int need = 0, extra = 0;
  bsa_status s = check_params(p, mode, param, &need);
  if (s != BSA_OK) return s;
  UnionOpts uo;
  if ((s = check_union(p, u, &uo, &extra)) != BSA_OK) return s;
  const int video = need - p->g.nb_text + extra;
  *kmax = (video < p->g.nb ? video : p->g.nb) + p->g.nb_text;
  return BSA_OK;
}

// Workspace of the forward: bsa_forward's (blocked tensors on SIMT plans,
// two summary arrays sized for centroids, the lists), plus two more
// centroid-sized arrays for box summaries (twice as wide), plus the K-block
// SICS and intra bit sets when the union has an intra part.
size_t forward_ws_bytes(const bsa_plan_s* p, int kmax, int est, bool intra) {
  size_t base = 0;
  bsa_workspace_size(const_cast<bsa_plan_s*>(p), kmax, nullptr, &base);
  if (est != bsa::kEstMean) base += 2 * round256(cent_bytes(p));
  if (intra) base += round256(bits_bytes(p)) + round256(sics_bytes(p));
  return base;
}

bsa_status forward_impl(bsa_plan_t p, const void* q, const void* k, const void* v,
                        bsa_select_mode mode, const double* param, const bsa_mask_union_t* u,
                        int kmax, void* o, int32_t* idx_out, int32_t* cnt_out, void* ws,
                        size_t ws_bytes, int32_t* dev_status, void* stream,
                        int est = bsa::kEstMean, PhaseTimer* timer = nullptr) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (est != bsa::kEstMean && est != bsa::kEstDsa && est != bsa::kEstDsa2)
    return fail(BSA_ERR_INVALID_ARG, "bad estimator %d", est);
  int need = 0;
  if ((s = union_kmax(p, mode, param, u, &need)) != BSA_OK) return s;
  if (kmax < need) return fail(BSA_ERR_INVALID_ARG, "kmax %d is below the %d entries a list can need", kmax, need);
  UnionOpts uo;
  int extra = 0;
  if ((s = check_union(p, u, &uo, &extra)) != BSA_OK) return s;
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const size_t need_ws = forward_ws_bytes(p, kmax, est, uo.intra);
  if (ws == nullptr || ws_bytes < need_ws)
    return fail(BSA_ERR_WORKSPACE, "forward needs %zu bytes of workspace, got %zu", need_ws, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  char* w = reinterpret_cast<char*>(ws);
  const size_t tb = p->attn_path == 1 ? 0 : round256(blk_bytes(p)), cb = round256(cent_bytes(p));
  void* q_blk = w; w += tb;
  void* k_blk = w; w += tb;
  void* v_blk = w; w += tb;
  void* o_blk = w; w += tb;
  float* qc = reinterpret_cast<float*>(w); w += cb;
  float* kc = reinterpret_cast<float*>(w); w += cb;
  int32_t* idx = reinterpret_cast<int32_t*>(w);
  w += round256((size_t)p->g.B * p->g.Hd * p->g.nb * kmax * sizeof(int32_t));
  int32_t* cnt = reinterpret_cast<int32_t*>(w);
  w += round256((size_t)p->g.B * p->g.Hd * p->g.nb * sizeof(int32_t));
  if (est != bsa::kEstMean) {
    // box summaries are twice as wide as centroids: Q's box takes the two
    // centroid slots, K's box the two extra slots
    kc = reinterpret_cast<float*>(w);
    w += 2 * cb;
  }
  float* k_sics = nullptr;
  uint32_t* bits = nullptr;
  if (uo.intra) {
    k_sics = reinterpret_cast<float*>(w); w += round256(sics_bytes(p));
    bits = reinterpret_cast<uint32_t*>(w); w += round256(bits_bytes(p));
  }
  if (idx_out) idx = idx_out;
  if (cnt_out) cnt = cnt_out;
  cudaStream_t st = (cudaStream_t)stream;
  const UnionOpts* up = u ? &uo : nullptr;
  if (p->attn_path == 1)
    return run_forward_fused(p, q, k, v, mode, param, kmax, o, idx, cnt, qc, kc, dev_status, st, up,
                             k_sics, bits, est, w, nullptr, timer);
  bsa::GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src[0] = q; a.src[1] = k; a.src[2] = v;
  a.dst[0] = q_blk; a.dst[1] = k_blk; a.dst[2] = v_blk;
  if (est == bsa::kEstMean) {
    a.cent[0] = qc; a.cent[1] = kc;
  } else {
    a.box[0] = qc; a.box[1] = kc;
  }
  a.sics[1] = k_sics;
  a.ntensors = 3;
  mark(timer);
  cudaError_t e = bsa::launch_permute(p->g, p->dtype == BSA_BF16, a, st);
  if (e != cudaSuccess) return cuda_fail(e, "permute kernel");
  mark(timer);
  if ((s = run_select(p, qc, kc, mode, param, kmax, idx, cnt, nullptr, st, up, k_sics, bits, est)) != BSA_OK)
    return s;
  mark(timer);
  if ((s = run_attention(p, q_blk, k_blk, v_blk, idx, cnt, kmax, o_blk, dev_status, st)) != BSA_OK) return s;
  mark(timer);
  s = bsa_unpermute(p, o_blk, o, stream);
  mark(timer);
  return s;
}

// Workspace of one scheme group of bsa_forward_grouped: its centroids, its
// lists and, with an intra part, its K-block SICS and bit sets.
size_t group_ws_bytes(const bsa_plan_s* p, int kmax, bool intra) {
  size_t w = 2 * round256(cent_bytes(p)) +
             round256((size_t)p->g.B * p->g.Hd * p->g.nb * kmax * sizeof(int32_t)) +
             round256((size_t)p->g.B * p->g.Hd * p->g.nb * sizeof(int32_t));
  if (intra) w += round256(sics_bytes(p)) + round256(bits_bytes(p));
  return w + pairing_bytes(p, kmax);
}

// Checks that the candidate plans describe the same problem (only the block
// shape differs), run on the tensor-core path, and that a head map fits.
bsa_status check_group_plans(const bsa_plan_t* plans, int n_plans) {
  if (plans == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL plan array");
  if (n_plans < 1 || n_plans > bsa::kMaxSchemes)
    return fail(BSA_ERR_INVALID_ARG, "n_plans = %d, must be in [1, %d]", n_plans, bsa::kMaxSchemes);
  for (int c = 0; c < n_plans; ++c) {
    bsa_status s = check_plan(plans[c]);
    if (s != BSA_OK) return s;
    const Geo& g = plans[c]->g;
    const Geo& g0 = plans[0]->g;
    if (g.B != g0.B || g.T != g0.T || g.H != g0.H || g.W != g0.W || g.Hd != g0.Hd ||
        g.D != g0.D || g.n_text != g0.n_text || plans[c]->dtype != plans[0]->dtype)
      return fail(BSA_ERR_INVALID_ARG,
                  "plan %d differs from plan 0 in more than the block shape", c);
    if (plans[c]->attn_path != 1)
      return fail(BSA_ERR_UNSUPPORTED, "grouped forward needs bf16 plans with 128-token blocks");
  }
  if ((long long)plans[0]->g.B * plans[0]->g.Hd > BSA_MAX_HEADS)
    return fail(BSA_ERR_UNSUPPORTED, "grouped forward needs batch * heads <= %d", BSA_MAX_HEADS);
  return BSA_OK;
}

}  // namespace

extern "C" {

int bsa_version(void) { return BSA_VERSION; }

const char* bsa_last_error_string(void) { return g_err.c_str(); }

bsa_status bsa_plan_create(bsa_plan_t* out, int batch, int T, int H, int W, int bf, int br, int bc,
                           int heads, int head_dim, int n_text, bsa_dtype dtype) {
  if (out == nullptr) return fail(BSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (batch < 1 || T < 1 || H < 1 || W < 1)
    return fail(BSA_ERR_INVALID_ARG, "batch and grid extents must be >= 1");
  if (bf < 1 || br < 1 || bc < 1) return fail(BSA_ERR_INVALID_ARG, "block extents must be >= 1");
  if (heads < 1 || heads > BSA_MAX_HEADS)
    return fail(BSA_ERR_INVALID_ARG, "heads must be in [1, %d]", BSA_MAX_HEADS);
  if (head_dim != 64 && head_dim != 128) return fail(BSA_ERR_INVALID_ARG, "head_dim must be 64 or 128");
  if (n_text < 0) return fail(BSA_ERR_INVALID_ARG, "n_text must be >= 0");
  if (dtype != BSA_F32 && dtype != BSA_BF16) return fail(BSA_ERR_INVALID_ARG, "bad dtype");
  const long long bs = (long long)bf * br * bc;
  if (bs > 256) return fail(BSA_ERR_INVALID_ARG, "block size bf*br*bc = %lld exceeds 256", bs);

  bsa_plan_s p;
  Geo& g = p.g;
  g.B = batch; g.T = T; g.H = H; g.W = W; g.bf = bf; g.br = br; g.bc = bc;
  g.Hd = heads; g.D = head_dim; g.n_text = n_text;
  g.nbt = (T + bf - 1) / bf; g.nby = (H + br - 1) / br; g.nbx = (W + bc - 1) / bc;
  const long long nb = (long long)g.nbt * g.nby * g.nbx;
  g.bs = (int)bs;
  g.nb_text = (int)((n_text + bs - 1) / bs);
  g.n_video = (long long)T * H * W;
  g.n_tot = g.n_video + n_text;
  const long long npad = (nb + g.nb_text) * bs;
  g.npad_tot = npad;
  if (nb > (1 << 24)) return fail(BSA_ERR_INVALID_ARG, "too many blocks");
  g.nb = (int)nb;
  if ((long long)batch * heads * npad >= (1ll << 31) || (long long)batch * g.n_tot * heads >= (1ll << 31))
    return fail(BSA_ERR_UNSUPPORTED, "problem exceeds 2^31 rows");
  // the selection kernel takes 8 query rows per CTA when 16 do not fit twice
  if (bsa::select_smem_bytes(g.nb, head_dim, 8) > 227 * 1024)
    return fail(BSA_ERR_UNSUPPORTED, "nb = %d video blocks exceeds the selection kernel's limit", g.nb);
  p.dtype = dtype;
  p.attn_path = (dtype == BSA_BF16 && bs == 128) ? 1 : 0;
  p.d_status = nullptr;
  p.d_masks = nullptr;
  p.wait_limit = 0;
  p.hold_load = 0;

  cudaError_t e = cudaGetDevice(&p.device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const int nbk = g.nb + g.nb_text;
  std::vector<uint32_t> masks((size_t)nbk * 4, 0u);
  if (bs <= 128)
    for (int j = 0; j < nbk; ++j)
      for (int s = 0; s < (int)bs; ++s)
        if (slot_token(g, j, s) >= 0) masks[(size_t)j * 4 + s / 32] |= 1u << (s % 32);
  e = cudaMalloc(&p.d_status, sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(status)");
  e = cudaMalloc(&p.d_masks, masks.size() * sizeof(uint32_t));
  if (e != cudaSuccess) { cudaFree(p.d_status); return cuda_fail(e, "cudaMalloc(masks)"); }
  if ((e = cudaMemset(p.d_status, 0, sizeof(int32_t))) != cudaSuccess ||
      (e = cudaMemcpy(p.d_masks, masks.data(), masks.size() * sizeof(uint32_t),
                      cudaMemcpyHostToDevice)) != cudaSuccess) {
    cudaFree(p.d_status);
    cudaFree(p.d_masks);
    return cuda_fail(e, "plan upload");
  }
  *out = new bsa_plan_s(p);
  return BSA_OK;
}

bsa_status bsa_plan_destroy(bsa_plan_t plan) {
  if (plan == nullptr) return BSA_OK;
  cudaFree(plan->d_status);
  cudaFree(plan->d_masks);
  delete plan;
  return BSA_OK;
}

bsa_status bsa_plan_get_info(bsa_plan_t p, bsa_plan_info_t* info) {
  if (p == nullptr || info == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL argument");
  const Geo& g = p->g;
  info->batch = g.B; info->T = g.T; info->H = g.H; info->W = g.W;
  info->bf = g.bf; info->br = g.br; info->bc = g.bc; info->heads = g.Hd; info->head_dim = g.D;
  info->n_text = g.n_text; info->dtype = (int)p->dtype;
  info->Tp = g.nbt * g.bf; info->Hp = g.nby * g.br; info->Wp = g.nbx * g.bc;
  info->nbt = g.nbt; info->nby = g.nby; info->nbx = g.nbx; info->nb = g.nb;
  info->nb_text = g.nb_text; info->bs = g.bs;
  info->n_video = g.n_video; info->n_tot = g.n_tot; info->npad_tot = g.npad_tot;
  info->attn_path = p->attn_path;
  return BSA_OK;
}

bsa_status bsa_kmax_for(bsa_plan_t p, bsa_select_mode mode, const double* param, int* kmax) {
  if (p == nullptr || kmax == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL argument");
  return check_params(p, mode, param, kmax);
}

bsa_status bsa_workspace_size(bsa_plan_t p, int kmax, size_t* select_ws, size_t* forward_ws) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (kmax < 1) return fail(BSA_ERR_INVALID_ARG, "kmax must be >= 1");
  const size_t cent = round256(cent_bytes(p));
  const size_t lists = round256((size_t)p->g.B * p->g.Hd * p->g.nb * kmax * sizeof(int32_t)) +
                       round256((size_t)p->g.B * p->g.Hd * p->g.nb * sizeof(int32_t));
  if (select_ws) *select_ws = 2 * cent;
  // The SIMT path stages blocked Q, K, V and O; the tensor-core path fuses the
  // layout transform into the attention loads and pairs the query tiles.
  if (forward_ws)
    *forward_ws = (p->attn_path == 1 ? pairing_bytes(p, kmax) : 4 * round256(blk_bytes(p))) +
                  2 * cent + lists;
  return BSA_OK;
}

bsa_status bsa_permute(bsa_plan_t p, const void* x, void* x_blk, float* centroids, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (!x || !x_blk) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(x_blk) || (centroids && !aligned16(centroids)))
    return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  bsa::GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src[0] = x; a.dst[0] = x_blk; a.cent[0] = centroids; a.ntensors = 1;
  cudaError_t e = bsa::launch_permute(p->g, p->dtype == BSA_BF16, a, (cudaStream_t)stream);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "permute kernel");
}

bsa_status bsa_permute_qkv(bsa_plan_t p, const void* q, const void* k, const void* v, void* q_blk,
                           void* k_blk, void* v_blk, float* q_cent, float* k_cent, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (!q || !k || !v || !q_blk || !k_blk || !v_blk) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  const void* ptrs[8] = {q, k, v, q_blk, k_blk, v_blk, q_cent, k_cent};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  bsa::GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src[0] = q; a.src[1] = k; a.src[2] = v;
  a.dst[0] = q_blk; a.dst[1] = k_blk; a.dst[2] = v_blk;
  a.cent[0] = q_cent; a.cent[1] = k_cent; a.cent[2] = nullptr;
  a.ntensors = 3;
  cudaError_t e = bsa::launch_permute(p->g, p->dtype == BSA_BF16, a, (cudaStream_t)stream);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "permute kernel");
}

bsa_status bsa_centroids(bsa_plan_t p, const void* q, const void* k, float* q_cent, float* k_cent,
                         void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if ((q_cent && !q) || (k_cent && !k)) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  const void* ptrs[4] = {q, k, q_cent, k_cent};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  return run_centroids(p, q, k, q_cent, k_cent, (cudaStream_t)stream);
}

bsa_status bsa_attention_orig(bsa_plan_t p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const int32_t* cnt, int kmax, void* o,
                              int32_t* dev_status, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  return run_attention_orig(p, q, k, v, idx, cnt, kmax, o, dev_status, (cudaStream_t)stream);
}

bsa_status bsa_unpermute(bsa_plan_t p, const void* o_blk, void* o, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (!o_blk || !o) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(o_blk) || !aligned16(o)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  bsa::GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src[0] = o_blk; a.dst[0] = o; a.ntensors = 1;
  cudaError_t e = bsa::launch_unpermute(p->g, p->dtype == BSA_BF16, a, (cudaStream_t)stream);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "unpermute kernel");
}

bsa_status bsa_select(bsa_plan_t p, const void* q_blk, const void* k_blk, bsa_select_mode mode,
                      const double* param, int kmax, int32_t* idx, int32_t* cnt, float* scores,
                      void* ws, size_t ws_bytes, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  int need = 0;
  if ((s = check_params(p, mode, param, &need)) != BSA_OK) return s;
  if (kmax < need) return fail(BSA_ERR_INVALID_ARG, "kmax %d is below the %d entries a list can need", kmax, need);
  if (!q_blk || !k_blk) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q_blk) || !aligned16(k_blk)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  size_t need_ws = 0;
  bsa_workspace_size(p, kmax, &need_ws, nullptr);
  if (ws == nullptr || ws_bytes < need_ws)
    return fail(BSA_ERR_WORKSPACE, "select needs %zu bytes of workspace, got %zu", need_ws, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  float* qc = reinterpret_cast<float*>(ws);
  float* kc = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round256(cent_bytes(p)));
  bsa::GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src[0] = q_blk; a.src[1] = k_blk; a.cent[0] = qc; a.cent[1] = kc; a.ntensors = 2;
  cudaError_t e = bsa::launch_pool(p->g, p->dtype == BSA_BF16, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "centroid kernel");
  return run_select(p, qc, kc, mode, param, kmax, idx, cnt, scores, (cudaStream_t)stream);
}

bsa_status bsa_select_centroids(bsa_plan_t p, const float* q_cent, const float* k_cent,
                                bsa_select_mode mode, const double* param, int kmax, int32_t* idx,
                                int32_t* cnt, float* scores, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  return run_select(p, q_cent, k_cent, mode, param, kmax, idx, cnt, scores, (cudaStream_t)stream);
}

bsa_status bsa_attention(bsa_plan_t p, const void* q_blk, const void* k_blk, const void* v_blk,
                         const int32_t* idx, const int32_t* cnt, int kmax, void* o_blk,
                         int32_t* dev_status, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  return run_attention(p, q_blk, k_blk, v_blk, idx, cnt, kmax, o_blk, dev_status, (cudaStream_t)stream);
}

bsa_status bsa_forward(bsa_plan_t p, const void* q, const void* k, const void* v,
                       bsa_select_mode mode, const double* param, int kmax, void* o,
                       int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes,
                       int32_t* dev_status, void* stream) {
  return forward_impl(p, q, k, v, mode, param, nullptr, kmax, o, idx_out, cnt_out, ws, ws_bytes,
                      dev_status, stream);
}

bsa_status bsa_forward_timed(bsa_plan_t p, const void* q, const void* k, const void* v,
                             bsa_select_mode mode, const double* param, int kmax, void* o,
                             int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream, bsa_timings_t* timings) {
  if (timings == nullptr) return fail(BSA_ERR_INVALID_ARG, "timings is NULL");
  std::memset(timings, 0, sizeof(*timings));
  PhaseTimer t;
  t.st = (cudaStream_t)stream;
  int made = 0;
  cudaError_t e = cudaSuccess;
  for (; made < 6 && e == cudaSuccess; ++made) e = cudaEventCreate(&t.ev[made]);
  if (e != cudaSuccess) made--;
  auto destroy = [&]() {
    for (int i = 0; i < made; ++i) cudaEventDestroy(t.ev[i]);
  };
  if (e != cudaSuccess) {
    destroy();
    return cuda_fail(e, "cudaEventCreate");
  }
  bsa_status s = forward_impl(p, q, k, v, mode, param, nullptr, kmax, o, idx_out, cnt_out, ws,
                              ws_bytes, dev_status, stream, bsa::kEstMean, &t);
  if (s == BSA_OK && t.err != cudaSuccess) s = cuda_fail(t.err, "cudaEventRecord");
  if (s == BSA_OK && t.n < 2) {   // nothing was launched: every phase took 0 ms
    destroy();
    return s;
  }
  if (s == BSA_OK && (e = cudaEventSynchronize(t.ev[t.n - 1])) != cudaSuccess) s = cuda_fail(e, "cudaEventSynchronize");
  if (s == BSA_OK) {
    float ms[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i + 1 < t.n && s == BSA_OK; ++i)
      if ((e = cudaEventElapsedTime(&ms[i], t.ev[i], t.ev[i + 1])) != cudaSuccess)
        s = cuda_fail(e, "cudaEventElapsedTime");
    if (s == BSA_OK) {
      if (p->attn_path == 1) {
        timings->summaries_ms = ms[0];
        timings->select_ms = ms[1];
        timings->pairing_ms = ms[2];
        timings->attention_ms = ms[3];
      } else {
        timings->summaries_ms = ms[0];   // permute with the fused centroids
        timings->select_ms = ms[1];
        timings->attention_ms = ms[2];
        timings->unpermute_ms = ms[3];
      }
      float total = 0.f;
      if ((e = cudaEventElapsedTime(&total, t.ev[0], t.ev[t.n - 1])) != cudaSuccess)
        s = cuda_fail(e, "cudaEventElapsedTime");
      timings->total_ms = total;
    }
  }
  destroy();
  return s;
}

bsa_status bsa_kmax_for_union(bsa_plan_t p, bsa_select_mode mode, const double* param,
                              const bsa_mask_union_t* u, int* kmax) {
  if (p == nullptr || kmax == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL plan or output");
  return union_kmax(p, mode, param, u, kmax);
}

bsa_status bsa_union_workspace_size(bsa_plan_t p, int kmax, const bsa_mask_union_t* u,
                                    size_t* select_ws, size_t* forward_ws) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "plan is NULL");
  UnionOpts uo;
  int extra = 0;
  bsa_status s = check_union(p, u, &uo, &extra);
  if (s != BSA_OK) return s;
  if (select_ws) *select_ws = uo.intra ? round256(bits_bytes(p)) : 0;
  if (forward_ws) *forward_ws = forward_ws_bytes(p, kmax, bsa::kEstMean, uo.intra);
  return BSA_OK;
}

bsa_status bsa_estimator_workspace_size(bsa_plan_t p, bsa_estimator est, int kmax,
                                        const bsa_mask_union_t* u, size_t* forward_ws) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (est != BSA_EST_MEAN && est != BSA_EST_DSA && est != BSA_EST_DSA2)
    return fail(BSA_ERR_INVALID_ARG, "bad estimator %d", (int)est);
  UnionOpts uo;
  int extra = 0;
  bsa_status s = check_union(p, u, &uo, &extra);
  if (s != BSA_OK) return s;
  if (forward_ws) *forward_ws = forward_ws_bytes(p, kmax, (int)est, uo.intra);
  return BSA_OK;
}

bsa_status bsa_box_summaries(bsa_plan_t p, const void* q, const void* k, float* q_box,
                             float* k_box, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if ((q_box && !q) || (k_box && !k)) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  const void* ptrs[4] = {q, k, q_box, k_box};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  return run_centroids(p, q, k, q_box, k_box, (cudaStream_t)stream, nullptr, true);
}

bsa_status bsa_select_box(bsa_plan_t p, bsa_estimator est, const float* q_box, const float* k_box,
                          bsa_select_mode mode, const double* param, const bsa_mask_union_t* u,
                          const float* intra_scores, int kmax, int32_t* idx, int32_t* cnt,
                          float* scores, void* ws, size_t ws_bytes, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (est != BSA_EST_DSA && est != BSA_EST_DSA2)
    return fail(BSA_ERR_INVALID_ARG, "bsa_select_box needs BSA_EST_DSA or BSA_EST_DSA2");
  int need = 0;
  if ((s = union_kmax(p, mode, param, u, &need)) != BSA_OK) return s;
  if (kmax < need) return fail(BSA_ERR_INVALID_ARG, "kmax %d is below the %d entries a list can need", kmax, need);
  UnionOpts uo;
  int extra = 0;
  if ((s = check_union(p, u, &uo, &extra)) != BSA_OK) return s;
  uint32_t* bits = nullptr;
  if (uo.intra) {
    if (intra_scores == nullptr) return fail(BSA_ERR_INVALID_ARG, "intra selection needs intra_scores");
    if (ws == nullptr || ws_bytes < bits_bytes(p))
      return fail(BSA_ERR_WORKSPACE, "union selection needs %zu bytes of workspace, got %zu",
                  round256(bits_bytes(p)), ws_bytes);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    bits = reinterpret_cast<uint32_t*>(ws);
  }
  return run_select(p, q_box, k_box, mode, param, kmax, idx, cnt, scores, (cudaStream_t)stream,
                    u ? &uo : nullptr, intra_scores, bits, (int)est);
}

bsa_status bsa_forward_estimator(bsa_plan_t p, const void* q, const void* k, const void* v,
                                 bsa_estimator est, bsa_select_mode mode, const double* param,
                                 const bsa_mask_union_t* u, int kmax, void* o, int32_t* idx_out,
                                 int32_t* cnt_out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                 void* stream) {
  return forward_impl(p, q, k, v, mode, param, u, kmax, o, idx_out, cnt_out, ws, ws_bytes,
                      dev_status, stream, (int)est);
}

bsa_status bsa_select_union(bsa_plan_t p, const float* q_cent, const float* k_cent,
                            bsa_select_mode mode, const double* param, const bsa_mask_union_t* u,
                            const float* intra_scores, int kmax, int32_t* idx, int32_t* cnt,
                            float* scores, void* ws, size_t ws_bytes, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  int need = 0;
  if ((s = union_kmax(p, mode, param, u, &need)) != BSA_OK) return s;
  if (kmax < need) return fail(BSA_ERR_INVALID_ARG, "kmax %d is below the %d entries a list can need", kmax, need);
  UnionOpts uo;
  int extra = 0;
  if ((s = check_union(p, u, &uo, &extra)) != BSA_OK) return s;
  uint32_t* bits = nullptr;
  if (uo.intra) {
    if (intra_scores == nullptr) return fail(BSA_ERR_INVALID_ARG, "intra selection needs intra_scores");
    if (ws == nullptr || ws_bytes < bits_bytes(p))
      return fail(BSA_ERR_WORKSPACE, "union selection needs %zu bytes of workspace, got %zu",
                  round256(bits_bytes(p)), ws_bytes);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    bits = reinterpret_cast<uint32_t*>(ws);
  }
  return run_select(p, q_cent, k_cent, mode, param, kmax, idx, cnt, scores, (cudaStream_t)stream,
                    &uo, intra_scores, bits);
}

bsa_status bsa_forward_union(bsa_plan_t p, const void* q, const void* k, const void* v,
                             bsa_select_mode mode, const double* param, const bsa_mask_union_t* u,
                             int kmax, void* o, int32_t* idx_out, int32_t* cnt_out, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream) {
  return forward_impl(p, q, k, v, mode, param, u, kmax, o, idx_out, cnt_out, ws, ws_bytes,
                      dev_status, stream);
}
bsa_status bsa_sics(bsa_plan_t p, const void* x, float* sics, void* stream) {
  bsa_plan_t plans[1] = {p};
  float* outs[1] = {sics};
  return bsa_aggregation_scores(plans, 1, x, outs, nullptr, nullptr, stream);
}

bsa_status bsa_aggregation_scores(const bsa_plan_t* plans, int n_plans, const void* x,
                                  float* const* sics, double* as, int32_t* choice, void* stream) {
  if (plans == nullptr || sics == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL plan or SICS array");
  if (n_plans < 1 || n_plans > bsa::kMaxSchemes)
    return fail(BSA_ERR_INVALID_ARG, "n_plans = %d, must be in [1, %d]", n_plans, bsa::kMaxSchemes);
  bsa::SchemeArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int c = 0; c < n_plans; ++c) {
    bsa_status s = check_plan(plans[c]);
    if (s != BSA_OK) return s;
    const Geo& g = plans[c]->g;
    const Geo& g0 = plans[0]->g;
    if (g.B != g0.B || g.T != g0.T || g.H != g0.H || g.W != g0.W || g.Hd != g0.Hd ||
        g.D != g0.D || g.n_text != g0.n_text || plans[c]->dtype != plans[0]->dtype)
      return fail(BSA_ERR_INVALID_ARG,
                  "candidate %d differs from candidate 0 in more than the block shape", c);
    if (sics[c] == nullptr && g.nb > 0) return fail(BSA_ERR_INVALID_ARG, "SICS output %d is NULL", c);
    a.g[c] = g;
    a.sics[c] = sics[c];
  }
  if (x == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(x)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  a.x = x;
  a.as = as;
  a.choice = choice;
  a.n = n_plans;
  const Geo& g0 = plans[0]->g;
  if ((long long)g0.B * g0.Hd > 65535)
    return fail(BSA_ERR_UNSUPPORTED, "batch * heads = %lld exceeds 65535", (long long)g0.B * g0.Hd);
  if ((long long)g0.B * g0.Hd == 0) return BSA_OK;
  cudaError_t e = bsa::launch_sics_schemes(a, plans[0]->dtype == BSA_BF16, (cudaStream_t)stream);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "SICS kernel");
}

bsa_status bsa_grouped_workspace_size(const bsa_plan_t* plans, int n_plans, const int* kmax_per_plan,
                                      const bsa_mask_union_t* u, size_t* forward_ws) {
  bsa_status s = check_group_plans(plans, n_plans);
  if (s != BSA_OK) return s;
  if (kmax_per_plan == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL kmax_per_plan");
  size_t total = 0;
  for (int c = 0; c < n_plans; ++c) {
    UnionOpts uo;
    int extra = 0;
    if ((s = check_union(plans[c], u, &uo, &extra)) != BSA_OK) return s;
    if (kmax_per_plan[c] < 1) return fail(BSA_ERR_INVALID_ARG, "kmax of plan %d must be >= 1", c);
    total += group_ws_bytes(plans[c], kmax_per_plan[c], uo.intra);
  }
  if (forward_ws) *forward_ws = total;
  return BSA_OK;
}

bsa_status bsa_forward_grouped(const bsa_plan_t* plans, int n_plans, const int32_t* head_plan,
                               const void* q, const void* k, const void* v, bsa_select_mode mode,
                               const double* param, const bsa_mask_union_t* u,
                               const int* kmax_per_plan, void* o, int32_t* const* idx_out,
                               int32_t* const* cnt_out, void* ws, size_t ws_bytes,
                               int32_t* dev_status, void* stream) {
  size_t need_ws = 0;
  bsa_status s = bsa_grouped_workspace_size(plans, n_plans, kmax_per_plan, u, &need_ws);
  if (s != BSA_OK) return s;
  const Geo& g0 = plans[0]->g;
  const int BH = g0.B * g0.Hd;
  if (head_plan == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL head_plan");
  for (int bh = 0; bh < BH; ++bh)
    if (head_plan[bh] < 0 || head_plan[bh] >= n_plans)
      return fail(BSA_ERR_INVALID_ARG, "head_plan[%d] = %d is not a plan index", bh, head_plan[bh]);
  for (int c = 0; c < n_plans; ++c) {
    int need = 0;
    if ((s = union_kmax(plans[c], mode, param, u, &need)) != BSA_OK) return s;
    if (kmax_per_plan[c] < need)
      return fail(BSA_ERR_INVALID_ARG, "kmax %d of plan %d is below the %d entries a list can need",
                  kmax_per_plan[c], c, need);
  }
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (ws == nullptr || ws_bytes < need_ws)
    return fail(BSA_ERR_WORKSPACE, "grouped forward needs %zu bytes of workspace, got %zu", need_ws, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  char* w = reinterpret_cast<char*>(ws);
  for (int c = 0; c < n_plans; ++c) {
    const bsa_plan_s* p = plans[c];
    const int kmax = kmax_per_plan[c];
    UnionOpts uo;
    int extra = 0;
    check_union(p, u, &uo, &extra);
    char* base = w;
    w += group_ws_bytes(p, kmax, uo.intra);
    bsa::HeadMap map;
    std::memset(&map, 0, sizeof(map));
    for (int bh = 0; bh < BH; ++bh)
      if (head_plan[bh] == c) map.bh[map.n++] = (uint8_t)bh;
    if (map.n == 0) continue;
    const size_t cb = round256(cent_bytes(p));
    float* qc = reinterpret_cast<float*>(base); base += cb;
    float* kc = reinterpret_cast<float*>(base); base += cb;
    int32_t* idx = reinterpret_cast<int32_t*>(base);
    base += round256((size_t)p->g.B * p->g.Hd * p->g.nb * kmax * sizeof(int32_t));
    int32_t* cnt = reinterpret_cast<int32_t*>(base);
    base += round256((size_t)p->g.B * p->g.Hd * p->g.nb * sizeof(int32_t));
    float* k_sics = nullptr;
    uint32_t* bits = nullptr;
    if (uo.intra) {
      k_sics = reinterpret_cast<float*>(base); base += round256(sics_bytes(p));
      bits = reinterpret_cast<uint32_t*>(base); base += round256(bits_bytes(p));
    }
    if (idx_out && idx_out[c]) idx = idx_out[c];
    if (cnt_out && cnt_out[c]) cnt = cnt_out[c];
    if ((s = run_forward_fused(p, q, k, v, mode, param, kmax, o, idx, cnt, qc, kc, dev_status, st,
                               u ? &uo : nullptr, k_sics, bits, bsa::kEstMean, base, &map)) != BSA_OK)
      return s;
  }
  return BSA_OK;
}

bsa_status bsa_pair_workspace_size(bsa_plan_t p, int kmax, size_t* bytes) {
  if (p == nullptr || bytes == nullptr) return fail(BSA_ERR_INVALID_ARG, "NULL plan or output");
  if (kmax < 1) return fail(BSA_ERR_INVALID_ARG, "kmax must be >= 1");
  *bytes = p->attn_path == 1 ? pairing_bytes(p, kmax) : 0;
  return BSA_OK;
}

bsa_status bsa_pair_tiles(bsa_plan_t p, const int32_t* idx, const int32_t* cnt, int kmax, void* ws,
                          size_t ws_bytes, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (p->attn_path != 1)
    return fail(BSA_ERR_UNSUPPORTED, "tile pairing serves bf16 plans with 128-token blocks");
  if (!bsa::pairing_supported(p->g))
    return fail(BSA_ERR_UNSUPPORTED, "tile pairing serves plans with at most 1536 video blocks (nb = %d)",
                p->g.nb);
  if (kmax < 1) return fail(BSA_ERR_INVALID_ARG, "kmax must be >= 1");
  if (p->g.nb > 0 && (!idx || !cnt)) return fail(BSA_ERR_INVALID_ARG, "NULL index list");
  if (ws == nullptr || ws_bytes < pairing_bytes(p, kmax))
    return fail(BSA_ERR_WORKSPACE, "pairing needs %zu bytes of workspace, got %zu",
                pairing_bytes(p, kmax), ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(BSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  int32_t* sched = nullptr;
  int32_t* lists = nullptr;
  return run_pairing(p, idx, cnt, kmax, reinterpret_cast<char*>(ws), &sched, &lists,
                     (cudaStream_t)stream, nullptr);
}

bsa_status bsa_attention_paired(bsa_plan_t p, const void* q, const void* k, const void* v,
                                const int32_t* idx, const int32_t* cnt, int kmax, void* ws,
                                size_t ws_bytes, void* o, int32_t* dev_status, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  if (p->attn_path != 1 || !bsa::pairing_supported(p->g))
    return fail(BSA_ERR_UNSUPPORTED, "paired attention serves bf16 plans with 128-token blocks and at "
                                     "most 1536 video blocks");
  if (ws == nullptr || ws_bytes < pairing_bytes(p, kmax))
    return fail(BSA_ERR_WORKSPACE, "paired attention needs the %zu-byte pairing workspace, got %zu",
                pairing_bytes(p, kmax), ws_bytes);
  const size_t bh = (size_t)p->g.B * p->g.Hd, pph = pairs_per_head(p->g);
  const char* w = reinterpret_cast<const char*>(ws) + round256(bsa::pair_scratch_bytes(p->g));
  const int32_t* sched = reinterpret_cast<const int32_t*>(w);
  const int32_t* lists = reinterpret_cast<const int32_t*>(w + round256(bh * pph * 4 * sizeof(int32_t)));
  return run_attention_orig(p, q, k, v, idx, cnt, kmax, o, dev_status, (cudaStream_t)stream,
                            nullptr, sched, lists, text_part_of(p, kmax, reinterpret_cast<char*>(ws)));
}

bsa_status bsa_check_status(bsa_plan_t p, void* stream) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t v = 0;
  if ((e = cudaMemcpy(&v, p->d_status, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "status read");
  if ((e = cudaMemset(p->d_status, 0, sizeof(v))) != cudaSuccess) return cuda_fail(e, "status reset");
  if (v == 0) return BSA_OK;
  return fail((bsa_status)v, "kernel reported status %d (%s)", v,
              v == BSA_ERR_TIMEOUT ? "a bounded wait ran out" : "an index list entry was out of range");
}

bsa_status bsa_plan_set_watchdog(bsa_plan_t p, long long wait_limit_cycles, int withhold_copy) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (wait_limit_cycles < 0 || withhold_copy < 0)
    return fail(BSA_ERR_INVALID_ARG, "wait limit and withheld copy must be >= 0");
  p->wait_limit = wait_limit_cycles;
  p->hold_load = withhold_copy;
  return BSA_OK;
}

}  // extern "C"

// Internal helpers for select_static.cu (C++ linkage, not part of the C ABI).
bsa_status bsa_internal_fail(bsa_status s, const char* msg) { return fail(s, "%s", msg); }

bsa_status bsa_internal_plan_sizes(bsa_plan_t p, const Geo** g, int* is_bf16, int* device) {
  bsa_status s = check_plan(p);
  if (s != BSA_OK) return s;
  *g = &p->g;
  *is_bf16 = p->dtype == BSA_BF16 ? 1 : 0;
  *device = p->device;
  return BSA_OK;
}
