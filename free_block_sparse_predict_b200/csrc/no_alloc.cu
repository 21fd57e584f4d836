// sparge_predict_mask_noalloc: the stage-1 predictor for callers that cannot
// allocate device memory when they call it and have no workspace to hand in
// (for example a plugin whose host framework owns every device buffer, or a
// serving loop that must not call the allocator after start-up).  The pooled
// block means and self-similarities that sparge_predict_mask keeps in the
// caller's workspace live here in one file-scope device array instead.
//
// The array is a fixed kNoAllocScratchBytes (32 MiB) per GPU; every GPU that
// loads the library holds it until the process exits.  All calls share it and
// it keeps the last call's contents: every region is completely rewritten by
// the pooling kernel before any kernel reads it, so nothing has to be cleared,
// and two calls whose kernels overlap on the GPU (different streams, no
// ordering between them) race on it.  The predictor's kernels have no
// device-side waits, so there is no status word to report.
#include <cstdint>
#include <mutex>

#include "sparge_internal.h"

namespace sparge {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device address).
cudaError_t scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[device] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return cudaSuccess;
}

}  // namespace
}  // namespace sparge

using namespace sparge;

extern "C" sparge_status_t sparge_predict_mask_noalloc(const sparge_params_t* p, const void* q,
                                                       const void* k, uint8_t* mask,
                                                       int32_t* kv_idx, int32_t* kv_cnt,
                                                       float* s_q, float* s_k,
                                                       cudaStream_t stream) {
  // the same parameter check, and so the same status codes, as sparge_predict_mask
  sparge_status_t st = check_params(p);
  if (st != SPARGE_OK) return st;
  if (p->qk_int8) return SPARGE_EUNSUPPORTED;  // the INT8 codes must outlive the call
  if (p->B == 0 || p->N == 0) return SPARGE_OK;
  if (q == nullptr || k == nullptr || mask == nullptr || kv_idx == nullptr || kv_cnt == nullptr)
    return SPARGE_EINVAL;
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(kv_idx) | reinterpret_cast<uintptr_t>(kv_cnt) |
                       reinterpret_cast<uintptr_t>(s_q) | reinterpret_cast<uintptr_t>(s_k);
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(k) & 15u) ||
      (a4 & 3u))
    return SPARGE_EINVAL;
  // the same carving as the workspace, restricted to the predictor's regions
  const WsLayout L = ws_layout(*p);
  if (L.s_k + align256(size_t(p->B) * p->Hkv * cdiv(p->N, p->bk) * 4) > kNoAllocScratchBytes)
    return SPARGE_EWORKSPACE;

  DeviceScope dev;
  if ((st = dev.enter(q)) != SPARGE_OK) return st;
  void* scratch = nullptr;
  if (scratch_address(dev.device(), &scratch) != cudaSuccess) return SPARGE_ECUDA;

  PredictPtrs x{};
  x.q = q;
  x.k = k;
  x.q_mean = ws_ptr<float>(scratch, L.q_mean);
  x.k_mean = ws_ptr<float>(scratch, L.k_mean);
  x.s_q = ws_ptr<float>(scratch, L.s_q);
  x.s_k = ws_ptr<float>(scratch, L.s_k);
  x.mask = mask;
  x.kv_idx = kv_idx;
  x.kv_cnt = kv_cnt;
  x.status = nullptr;  // the predictor's kernels have no device-side waits to report
  if (launch_predict(*p, x, stream) != cudaSuccess) return SPARGE_ECUDA;
  const int64_t Tm = cdiv(p->N, p->bq), Tn = cdiv(p->N, p->bk);
  if (s_q != nullptr && cudaMemcpyAsync(s_q, x.s_q, size_t(p->B) * p->Hq * Tm * 4,
                                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return SPARGE_ECUDA;
  if (s_k != nullptr && cudaMemcpyAsync(s_k, x.s_k, size_t(p->B) * p->Hkv * Tn * 4,
                                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return SPARGE_ECUDA;
  return SPARGE_OK;
}
