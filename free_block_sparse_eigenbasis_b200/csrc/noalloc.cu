// sparsepr_route_noalloc: the routing call without a caller workspace.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that must not synchronise the device (cudaMalloc can), processes that
// reserve all device memory up front in their own pool, and hosts whose
// memory plan is fixed before the first call. This entry point computes the
// routes of sparsepr_route with the same kernels (group means, fp64 score
// GEMM, top-k), so its routes are those of sparsepr_route bit for bit; its
// scratch (the group means and the block scores) lives in one file-scope
// device array of fixed size instead of the caller's workspace, and it
// allocates nothing.
//
//   * Scratch: kRouteScratchBytes (8 MiB) per GPU, held until the process
//     exits. Under CUDA's default lazy module loading the array is committed
//     when the first call on a device looks its address up (so that first
//     call can allocate and synchronise); with eager loading
//     (CUDA_MODULE_LOADING=EAGER) it is committed when the library is
//     loaded. Heads are processed in chunks that fit; one head needs
//     ((Cq + Ck) d + Cq Ck) * 8 bytes, and parameters whose single head does
//     not fit are rejected with SPARSEPR_ERR_WORKSPACE.
//   * Set-up: the first call on each device looks up the array's device
//     address (cudaGetSymbolAddress) with that device current. Make that
//     first call before any stream capture.
//   * Every call shares the one array and it keeps the last call's
//     contents; each call overwrites all the scratch it reads, so nothing
//     needs clearing. Calls whose work overlaps on the GPU (other streams,
//     other host threads) race on the array: order them on one stream.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr size_t kRouteScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace spr

using namespace spr;

extern "C" sparsepr_status sparsepr_route_noalloc(const void* qp, const void* kp,
                                                  sparsepr_dtype dt, const sparsepr_params* p,
                                                  const int32_t* off_q, const int32_t* off_k,
                                                  int32_t* csr, int32_t* k_per_head,
                                                  void* stream) {
  if (sparsepr_workspace_bytes(p) == 0) {
    if (p && p->keep && (p->d != 64 && p->d != 128)) return SPARSEPR_ERR_UNSUPPORTED;
    return SPARSEPR_ERR_INVALID_ARG;
  }
  if (dt != SPARSEPR_BF16 && dt != SPARSEPR_F32) return SPARSEPR_ERR_UNSUPPORTED;
  if (!qp || !kp || !off_q || !off_k || !csr || !k_per_head) return SPARSEPR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qp) & 15) || (reinterpret_cast<uintptr_t>(kp) & 15))
    return SPARSEPR_ERR_INVALID_ARG;  // rows are read with 16-byte loads, as in sparsepr_route
  const int H = p->H, N = p->N, d = p->d, Ck = p->Ck, Cq = p->Cq;
  const int text = p->n_text > 0 ? 1 : 0;  // the text groups are kept outside the budget
  const int oq = Cq + text + 1, ok = Ck + text + 1;  // offsets per head
  const size_t means_head = (static_cast<size_t>(Cq) + Ck) * d * sizeof(double);
  const size_t scores_head = static_cast<size_t>(Cq) * Ck * sizeof(double);
  if (means_head + scores_head > kRouteScratchBytes) return SPARSEPR_ERR_WORKSPACE;
  // heads per chunk: their group means plus the block scores of at least one head
  const int chunk = static_cast<int>((kRouteScratchBytes - scores_head) / means_head);
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const double scale = p->scale > 0.0 ? p->scale : 1.0 / sqrt(static_cast<double>(d));
  const int kind = (dt == SPARSEPR_BF16) ? kXbf16 : kXf32;
  const size_t eb = (dt == SPARSEPR_BF16) ? 2 : 4;
  int32_t kh[SPARSEPR_MAX_HEADS];
  int kmax = 1;
  for (int h = 0; h < H; ++h) {
    kh[h] = keep_budget(p->keep[h], Ck);
    if (kh[h] > kmax) kmax = kh[h];
  }
  if (launch_write_k(kh, H, k_per_head, st) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  double* cq = static_cast<double*>(base);
  for (int h0 = 0; h0 < H; h0 += chunk) {
    const int hc = (H - h0 < chunk) ? (H - h0) : chunk;
    double* ckr = cq + static_cast<size_t>(hc) * Cq * d;
    double* scores = ckr + static_cast<size_t>(hc) * Ck * d;
    const size_t scores_bytes = kRouteScratchBytes - static_cast<size_t>(hc) * means_head;
    const size_t head_elems = static_cast<size_t>(N) * d;
    const char* qh = static_cast<const char*>(qp) + h0 * head_elems * eb;
    const char* kh0 = static_cast<const char*>(kp) + h0 * head_elems * eb;
    if (launch_range_mean(qh, kind, hc, N, d, off_q + static_cast<size_t>(h0) * oq, Cq, oq, cq,
                          st) != cudaSuccess ||
        launch_range_mean(kh0, kind, hc, N, d, off_k + static_cast<size_t>(h0) * ok, Ck, ok, ckr,
                          st) != cudaSuccess ||
        launch_route_gemm(cq, ckr, hc, Cq, Ck, d, scale, k_per_head + h0, kmax, scores,
                          scores_bytes, csr + static_cast<size_t>(h0) * Cq * kmax,
                          st) != cudaSuccess)
      return SPARSEPR_ERR_CUDA;
  }
  return SPARSEPR_OK;
}
