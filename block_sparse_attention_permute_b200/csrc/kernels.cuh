// kernels.cuh — argument blocks and launchers of the libbsa kernels
// (internal; the public interface is include/bsa.h).
#pragma once
#include "common.cuh"

namespace bsa {

// The (batch, head) pairs one launch covers: n = 0 means all B * Hd pairs in
// order; otherwise the pairs bh[0..n), bh = b * Hd + h (B * Hd <= 256).  This
// is how heads that share a blocking scheme are grouped into one launch.
struct HeadMap {
  int n;
  uint8_t bh[BSA_MAX_HEADS];
};
__host__ __device__ __forceinline__ int map_count(const HeadMap& m, int all) { return m.n ? m.n : all; }
__host__ __device__ __forceinline__ int map_bh(const HeadMap& m, int x) { return m.n ? (int)m.bh[x] : x; }

struct GatherArgs {
  const void* src[3];
  void* dst[3];      // unused in kPool
  float* cent[3];    // optional centroid outputs (kPermute, kPool)
  float* sics[3];    // optional SICS outputs [B, Hd, nb] (kPermute, kPool, kPoolOrig)
  float* box[3];     // optional box summaries [B, Hd, nb, D, 2] = (max, min) (same modes)
  int ntensors;
  HeadMap map;
};

// Aggregation evaluation of up to kMaxSchemes candidate blocking schemes of
// one tensor in the original layout (every g[c] shares B, T, H, W, Hd, D,
// n_text; only the block shape differs).
constexpr int kMaxSchemes = 8;
struct SchemeArgs {
  Geo g[kMaxSchemes];
  float* sics[kMaxSchemes];   // [B, Hd, nb_c] per candidate
  const void* x;              // [B, Ntot, Hd, D]
  double* as;                 // [n, B, Hd] or null
  int32_t* choice;            // [B, Hd] or null
  int n;
};

// Inter-estimators of the selection: MEAN dots the centroids; DSA dots
// (c+, c-) of the query box centre c with the key box (max, min); DSA2 sums,
// per dimension, the largest corner product of the two boxes.
enum Estimator { kEstMean = 0, kEstDsa = 1, kEstDsa2 = 2 };

struct SelectArgs {
  const float* qc;   // [B, Hd, nb, D] centroids, or [B, Hd, nb, D, 2] boxes
  const float* kc;   // same layout as qc
  int32_t* idx;      // [B, Hd, nb, kmax]
  int32_t* cnt;      // [B, Hd, nb]
  float* scores;     // [B, Hd, nb, nb] or null
  int kmax;
  int mode;          // 0 top-k, 1 top-p
  int est;           // Estimator
  float scale;       // 1/sqrt(D) rounded to fp32
  double param[BSA_MAX_HEADS];  // k (held in a double) or tau, per head
  // Mask union (video key blocks added to every list of a head):
  int win_left, win_right;      // j in [i - left, i + right]; < 0 = unbounded; both < 0 = none
  long long sink_tokens;        // blocks holding any of the first sink_tokens tokens
  const uint32_t* intra_bits;   // [B, Hd, nbw] selected key blocks, or null
  uint32_t* list_bits;          // [B * Hd, nb, nbw] out: each list's video blocks as a bit set, or null
  HeadMap map;
};

// Selection on per-key-block intra scores (one warp per (b, h)).
struct IntraArgs {
  const float* scores;          // [B, Hd, nb]
  uint32_t* bits;               // [B, Hd, nbw], nbw = ceil(nb / 32)
  int mode;                     // 0 top-k, 1 top-p
  double param[BSA_MAX_HEADS];  // k (held in a double) or tau per head; <= 0 = none
  HeadMap map;
};

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  const int32_t* idx;     // [B, Hd, nb, kmax]
  const int32_t* cnt;     // [B, Hd, nb]
  const uint32_t* masks;  // [(nb + nb_text) * 4] slot validity bits (bs == 128 only)
  int32_t* status;        // device status word
  int kmax;
  long long wait_limit;   // bound of every in-kernel wait, SM cycles (0 = kWaitLimitDefault)
  int hold_load;          // test hook: n > 0 = CTA 0 never issues its n-th K/V copy; 0 = off
  float scale;            // 1/sqrt(D)
  float scale_log2;       // log2(e)/sqrt(D)
  HeadMap map;
  // Paired schedule (original-layout path, one batch element per launch), or
  // null for the plain order (tiles 2x and 2x+1).  Entry (h, t) of a head,
  // t < text_pairs for its text tiles, then its video pairs:
  //   pair_sched[(h * pairs_per_head + t) * 4 + {0,1,2}] = {i0, i1 (-1 = none), c}
  //   pair_lists[((h * pairs_per_head + t) * 2 + x) * kmax + s] = block of step s
  // The first c steps of both tiles visit the same key blocks (their K and V
  // tiles are fetched once); video tiles read their lists from pair_lists.
  const int32_t* pair_sched;
  const int32_t* pair_lists;
  int pairs_per_head, text_pairs;
  // Text pairs of the paired schedule split into text_chunks key chunks of
  // text_chunk_len blocks; a chunk's partial rows go to
  //   part[((((bh * nb_text + (i - nb)) * text_chunks + c) * 128 + r) * (D + 4) + d]
  //   d < D: unnormalised O, d = D: running max (log2 units), d = D + 1: row sum
  float* part;
  int text_chunks, text_chunk_len;
  // divisors of the per-copy block coordinates (nbx, nby, Hd), so that the
  // copy-issuing thread divides without the MUFU unit
  FastDiv div_nbx, div_nby, div_hd;
};

// Merge of the text rows' key-chunk partials into the output (original
// layout, one batch element per launch).
struct MergeArgs {
  const float* part;      // as AttnArgs::part
  void* o;                // [Ntot, Hd, D] of the batch element
  int text_chunks;
  HeadMap map;            // heads of the launch (n = 0: all)
};

// Pairing of the query tiles of each (b, h) into CTA pairs that share key
// blocks (pair.cu).
struct PairArgs {
  const int32_t* idx;     // [B, Hd, nb, kmax] lists (ascending video blocks, then text)
  const int32_t* cnt;     // [B, Hd, nb]
  uint32_t* bits;         // [B * Hd, nb, nbw] scratch: list bit sets
  uint16_t* cand;         // [B * Hd, nb, 8] scratch: best partners by |L_i & L_j|
  int32_t* sched;         // [B * Hd, pairs_per_head, 4] out
  int32_t* lists;         // [B * Hd, pairs_per_head, 2, kmax] out
  int kmax;
  int pairs_per_head, text_pairs;
  int bits_ready;         // the bit sets were written by the selection (no bit-set pass)
  HeadMap map;            // pairs of (b, h) to pair up (n = 0: all)
};

// TMA tensor maps of one attention launch: q/k/v cover the blocked tensors
// (2D) or the video tokens of the original layout (5D); qt/kt/vt cover the
// text tokens of the original layout (3D, unused otherwise).
struct TileMaps {
  CUtensorMap q, k, v, qt, kt, vt;
};

// permute.cu
cudaError_t launch_permute(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st);
cudaError_t launch_unpermute(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st);
cudaError_t launch_pool(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st);
cudaError_t launch_sics_schemes(const SchemeArgs& a, bool is_bf16, cudaStream_t st);
// select.cu
size_t select_smem_bytes(int nb, int D, int rows = 16, int kpt = 2);   // rows: query blocks per CTA; kpt: keys per thread
cudaError_t launch_select(const Geo& g, const SelectArgs& a, cudaStream_t st);
cudaError_t launch_intra_select(const Geo& g, const IntraArgs& a, cudaStream_t st);
// pair.cu
size_t pair_scratch_bytes(const Geo& g);
// Tile pairing serves plans with at most 32 * 48 = 1536 video blocks (bit sets
// of 48 words); larger plans run the attention unpaired.
bool pairing_supported(const Geo& g);
cudaError_t launch_pairing(const Geo& g, const PairArgs& a, cudaStream_t st);
// attn.cu
size_t attn_tc_smem_bytes(int D);
cudaError_t launch_attn_simt(const Geo& g, bool is_bf16, const AttnArgs& a, cudaStream_t st);
cudaError_t launch_attn_tc(const Geo& g, const AttnArgs& a, const TileMaps& maps, cudaStream_t st);
cudaError_t launch_attn_tc_orig(const Geo& g, const AttnArgs& a, const TileMaps& maps,
                                cudaStream_t st);
cudaError_t launch_text_merge(const Geo& g, const MergeArgs& a, cudaStream_t st);
cudaError_t launch_pool_orig(const Geo& g, bool is_bf16, const GatherArgs& a, cudaStream_t st);

}  // namespace bsa
