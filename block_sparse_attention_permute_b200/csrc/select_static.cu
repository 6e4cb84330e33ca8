// select_static.cu — bsa_select_static: the index search of bsa_select with
// its scratch memory (the fp32 Q and K centroids) held in a fixed device
// array that this file defines, so the call allocates nothing.
//
// Some callers cannot hand us a workspace or let us call cudaMalloc: engines
// and plugin hosts that plan every byte of device memory before serving
// starts and forbid allocation afterwards, and hot loops that cannot afford
// cudaMalloc's implicit device-wide synchronisation or its failure under
// fragmentation.  They pay instead with a fixed 16 MiB array that every GPU
// holds from the moment the library is loaded until the process exits.
//
// Set-up: the first call on each device looks up that device's copy of the
// array with cudaGetSymbolAddress (with that device current) and caches the
// address together with the id of the current context; a later call in
// another context (after a device reset, say) looks it up again.  Make the
// first call on a device before any stream capture begins.
// Sharing: all calls on a device use the same array and it keeps the last
// call's contents.  Every centroid is rewritten by each call before it is
// read, so nothing needs clearing, but calls whose kernels overlap on the
// GPU (for example on two streams) race on the array.
#include <cstring>
#include <mutex>

#include "bsa.h"
#include "kernels.cuh"

// Largest centroid scratch a call may need: 2 * B * Hd * nb * D * 4 bytes.
#define BSA_STATIC_SCRATCH_BYTES (16u << 20)

static __device__ __align__(256) unsigned char g_select_scratch[BSA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};   // context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (0 if the driver
// cannot tell): a device reset or a re-created primary context gets a new id,
// and with it a new copy of the array at a new address.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's copy of g_select_scratch (the host-side
// name is only a stand-in and must never be handed to a kernel).  Looked up
// once per device and context; looked up again whenever the current context
// differs from the one the cached address came from (or cannot be told).
cudaError_t scratch_for_device(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

// Defined in api.cu (internal, not part of the C ABI).
bsa_status bsa_internal_fail(bsa_status s, const char* msg);
bsa_status bsa_internal_plan_sizes(bsa_plan_t plan, const Geo** g, int* is_bf16, int* device);

extern "C" bsa_status bsa_select_static(bsa_plan_t plan, const void* q_blk, const void* k_blk,
                                        bsa_select_mode mode, const double* param_per_head,
                                        int kmax, int32_t* idx, int32_t* cnt, float* scores,
                                        void* stream) {
  const Geo* g = nullptr;
  int is_bf16 = 0, device = -1;
  bsa_status s = bsa_internal_plan_sizes(plan, &g, &is_bf16, &device);
  if (s != BSA_OK) return s;
  if (!q_blk || !k_blk || !idx || !cnt)
    return bsa_internal_fail(BSA_ERR_INVALID_ARG, "NULL tensor or list pointer");
  if ((reinterpret_cast<uintptr_t>(q_blk) & 15u) || (reinterpret_cast<uintptr_t>(k_blk) & 15u))
    return bsa_internal_fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const size_t cent = (size_t)g->B * g->Hd * g->nb * g->D * sizeof(float);
  const size_t cent_padded = (cent + 255) & ~size_t(255);
  if (2 * cent_padded > BSA_STATIC_SCRATCH_BYTES)
    return bsa_internal_fail(BSA_ERR_UNSUPPORTED,
                             "bsa_select_static: the centroids of this plan need more than the "
                             "16 MiB static scratch (2 * batch * heads * nb * head_dim * 4 bytes); "
                             "use bsa_select with a workspace");
  void* base = nullptr;
  cudaError_t e = scratch_for_device(device, &base);
  if (e != cudaSuccess) return bsa_internal_fail(BSA_ERR_CUDA, cudaGetErrorString(e));
  float* qc = reinterpret_cast<float*>(base);
  float* kc = reinterpret_cast<float*>(reinterpret_cast<char*>(base) + cent_padded);
  // Validate the selection parameters before anything is launched.
  int need = 0;
  if ((s = bsa_kmax_for(plan, mode, param_per_head, &need)) != BSA_OK) return s;
  if (kmax < need) return bsa_internal_fail(BSA_ERR_INVALID_ARG, "kmax is below what a list can need");
  bsa::GatherArgs a;
  memset(&a, 0, sizeof(a));
  a.src[0] = q_blk; a.src[1] = k_blk; a.cent[0] = qc; a.cent[1] = kc; a.ntensors = 2;
  e = bsa::launch_pool(*g, is_bf16 != 0, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return bsa_internal_fail(BSA_ERR_CUDA, cudaGetErrorString(e));
  return bsa_select_centroids(plan, qc, kc, mode, param_per_head, kmax, idx, cnt, scores, stream);
}
