// extern "C" entry points of libsparge: argument validation, workspace
// carving and launches on the caller's stream.  See include/sparge.h.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "sparge_internal.h"

using namespace sparge;

namespace {

// Largest key-block count the stage-1 select kernel keeps in shared memory.
constexpr int64_t kMaxTn = 5952;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool empty_problem(const sparge_params_t* p) { return p->B == 0 || p->N == 0; }

sparge_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SPARGE_OK;
  if (e == cudaErrorNotSupported) return SPARGE_EUNSUPPORTED;
  return SPARGE_ECUDA;
}

int elem_size(sparge_dtype_t t) { return t == SPARGE_F32 ? 4 : 2; }

}  // namespace

namespace sparge {

sparge_status_t check_params(const sparge_params_t* p) {
  if (p == nullptr) return SPARGE_EINVAL;
  if (p->B < 0 || p->N < 0 || p->Hq < 1 || p->Hkv < 1 || p->d < 1) return SPARGE_EINVAL;
  if (p->Hq % p->Hkv != 0) return SPARGE_EINVAL;
  if (!(p->tau > 0.f) || std::isnan(p->tau)) return SPARGE_EINVAL;
  if (std::isnan(p->theta) || std::isnan(p->lambda) || p->lambda > 0.f) return SPARGE_EINVAL;
  if (!std::isfinite(p->scale) || !(p->scale > 0.f)) return SPARGE_EINVAL;
  if ((p->causal != 0 && p->causal != 1) || (p->qk_int8 != 0 && p->qk_int8 != 1))
    return SPARGE_EINVAL;
  if (p->io_dtype != SPARGE_F16 && p->io_dtype != SPARGE_BF16) return SPARGE_EINVAL;
  if (p->o_dtype != p->io_dtype && p->o_dtype != SPARGE_F32) return SPARGE_EINVAL;
  if (p->d != 64 && p->d != 128) return SPARGE_EUNSUPPORTED;
  if (p->bq != 128 || p->bk != 64) return SPARGE_EUNSUPPORTED;
  if (p->qk_int8 && p->d != 128) return SPARGE_EUNSUPPORTED;
  if (cdiv(p->N, p->bk) > kMaxTn) return SPARGE_EUNSUPPORTED;
  if (p->B > 65535 || p->Hq > 65535) return SPARGE_EUNSUPPORTED;
  const int64_t tiles = int64_t(p->B) * p->Hq * cdiv(p->N, p->bq);
  if (tiles > int64_t(INT32_MAX)) return SPARGE_EUNSUPPORTED;
  return SPARGE_OK;
}

}  // namespace sparge

extern "C" {

size_t sparge_workspace_bytes(const sparge_params_t* p) {
  if (check_params(p) != SPARGE_OK) return 0;
  return ws_layout(*p).total;
}

size_t sparge_hilbert_workspace_bytes(int32_t T, int32_t Hg, int32_t Wg) {
  return hilbert_ws_bytes(T, Hg, Wg);
}

sparge_status_t sparge_hilbert_index(int32_t N, int32_t prefix_len, int32_t T, int32_t Hg,
                                     int32_t Wg, int32_t* perm, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  if (N < 0 || prefix_len < 0 || T < 1 || Hg < 1 || Wg < 1) return SPARGE_EINVAL;
  if (int64_t(T) * Hg * Wg + prefix_len > N) return SPARGE_EINVAL;
  const size_t need = hilbert_ws_bytes(T, Hg, Wg);
  if (need == 0) return SPARGE_EUNSUPPORTED;
  if (N == 0) return SPARGE_OK;
  if (perm == nullptr || ws == nullptr || (reinterpret_cast<uintptr_t>(perm) & 3u)) return SPARGE_EINVAL;
  if (ws_bytes < need) return SPARGE_EWORKSPACE;
  DeviceScope dev;
  sparge_status_t st = dev.enter(perm);
  if (st != SPARGE_OK) return st;
  return from_cuda(launch_hilbert_index(N, prefix_len, T, Hg, Wg, perm, ws, stream));
}

static sparge_status_t permute_common(const void* src, void* dst, int32_t B, int32_t H,
                                      int32_t N, int32_t d, sparge_dtype_t dtype,
                                      const int32_t* perm, bool inverse, cudaStream_t stream) {
  if (B < 0 || H < 0 || N < 0 || d < 1) return SPARGE_EINVAL;
  if (dtype != SPARGE_F16 && dtype != SPARGE_BF16 && dtype != SPARGE_F32) return SPARGE_EINVAL;
  const int64_t row_bytes = int64_t(d) * elem_size(dtype);
  if (row_bytes % 16 != 0) return SPARGE_EUNSUPPORTED;
  if (int64_t(B) * H > 65535) return SPARGE_EUNSUPPORTED;
  if (int64_t(B) * H * N == 0) return SPARGE_OK;
  if (src == nullptr || dst == nullptr || perm == nullptr) return SPARGE_EINVAL;
  if (!aligned16(src) || !aligned16(dst)) return SPARGE_EINVAL;
  const int64_t bytes = int64_t(B) * H * N * row_bytes;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  if (s0 < d0 + bytes && d0 < s0 + bytes) return SPARGE_EINVAL;  // overlap
  DeviceScope dev;
  sparge_status_t st = dev.enter(dst);
  if (st != SPARGE_OK) return st;
  return from_cuda(
      launch_permute_rows(src, dst, int64_t(B) * H, N, int32_t(row_bytes), perm, inverse, stream));
}

sparge_status_t sparge_hilbert_permute(const void* x, void* y, int32_t B, int32_t H, int32_t N,
                                       int32_t d, sparge_dtype_t dtype, const int32_t* perm,
                                       cudaStream_t stream) {
  return permute_common(x, y, B, H, N, d, dtype, perm, false, stream);
}

sparge_status_t sparge_inverse_permute(const void* y, void* x, int32_t B, int32_t H, int32_t N,
                                       int32_t d, sparge_dtype_t dtype, const int32_t* perm,
                                       cudaStream_t stream) {
  return permute_common(y, x, B, H, N, d, dtype, perm, true, stream);
}

enum : int { kStagePool = 1, kStageSelect = 2 };

// The predictor's entry points share one argument check; `stages` says which
// half runs (the pooled block statistics travel through the workspace).
static sparge_status_t predict_common(int stages, const sparge_params_t* p, const void* q,
                                      const void* k, uint8_t* mask, int32_t* kv_idx,
                                      int32_t* kv_cnt, float* s_q, float* s_k, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
  sparge_status_t st = check_params(p);
  if (st != SPARGE_OK) return st;
  if (empty_problem(p)) return SPARGE_OK;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPARGE_EINVAL;
  if (stages & kStagePool) {
    if (q == nullptr || k == nullptr || !aligned16(q) || !aligned16(k)) return SPARGE_EINVAL;
  }
  if (stages & kStageSelect) {
    if (mask == nullptr || kv_idx == nullptr || kv_cnt == nullptr) return SPARGE_EINVAL;
    if ((reinterpret_cast<uintptr_t>(kv_idx) & 3u) || (reinterpret_cast<uintptr_t>(kv_cnt) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_q) & 3u) || (reinterpret_cast<uintptr_t>(s_k) & 3u))
      return SPARGE_EINVAL;
  }
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.total) return SPARGE_EWORKSPACE;
  DeviceScope dev;
  if ((st = dev.enter((stages & kStagePool) ? q : ws)) != SPARGE_OK) return st;
  PredictPtrs x{};
  x.q = q;
  x.k = k;
  x.q_mean = ws_ptr<float>(ws, L.q_mean);
  x.k_mean = ws_ptr<float>(ws, L.k_mean);
  x.s_q = ws_ptr<float>(ws, L.s_q);
  x.s_k = ws_ptr<float>(ws, L.s_k);
  if (p->qk_int8) {
    x.q_codes = ws_ptr<int8_t>(ws, L.q_codes);
    x.k_codes = ws_ptr<int8_t>(ws, L.k_codes);
    x.dq = ws_ptr<float>(ws, L.dq);
    x.dk = ws_ptr<float>(ws, L.dk);
    x.kbar = ws_ptr<float>(ws, L.kbar);
    x.ksum64 = ws_ptr<double>(ws, L.k_sum64);
  }
  x.mask = mask;
  x.kv_idx = kv_idx;
  x.kv_cnt = kv_cnt;
  x.status = ws_ptr<int32_t>(ws, L.status);
  if (stages & kStagePool) {
    const cudaError_t e = launch_predict_pool(*p, x, stream);
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (!(stages & kStageSelect)) return SPARGE_OK;
  const cudaError_t e = launch_predict_select(*p, x, stream);
  if (e != cudaSuccess) return from_cuda(e);
  const int64_t Tm = cdiv(p->N, p->bq), Tn = cdiv(p->N, p->bk);
  if (s_q != nullptr &&
      cudaMemcpyAsync(s_q, x.s_q, size_t(p->B) * p->Hq * Tm * 4, cudaMemcpyDeviceToDevice,
                      stream) != cudaSuccess)
    return SPARGE_ECUDA;
  if (s_k != nullptr &&
      cudaMemcpyAsync(s_k, x.s_k, size_t(p->B) * p->Hkv * Tn * 4, cudaMemcpyDeviceToDevice,
                      stream) != cudaSuccess)
    return SPARGE_ECUDA;
  return SPARGE_OK;
}

sparge_status_t sparge_predict_mask(const sparge_params_t* p, const void* q, const void* k,
                                    uint8_t* mask, int32_t* kv_idx, int32_t* kv_cnt, float* s_q,
                                    float* s_k, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return predict_common(kStagePool | kStageSelect, p, q, k, mask, kv_idx, kv_cnt, s_q, s_k, ws,
                        ws_bytes, stream);
}

sparge_status_t sparge_predict_pool(const sparge_params_t* p, const void* q, const void* k,
                                    void* ws, size_t ws_bytes, cudaStream_t stream) {
  return predict_common(kStagePool, p, q, k, nullptr, nullptr, nullptr, nullptr, nullptr, ws,
                        ws_bytes, stream);
}

sparge_status_t sparge_predict_select(const sparge_params_t* p, uint8_t* mask, int32_t* kv_idx,
                                      int32_t* kv_cnt, float* s_q, float* s_k, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
  return predict_common(kStageSelect, p, nullptr, nullptr, mask, kv_idx, kv_cnt, s_q, s_k, ws,
                        ws_bytes, stream);
}

sparge_status_t sparge_mask_compact(const sparge_params_t* p, const uint8_t* mask,
                                    int32_t* kv_idx, int32_t* kv_cnt, cudaStream_t stream) {
  sparge_status_t st = check_params(p);
  if (st != SPARGE_OK) return st;
  if (empty_problem(p)) return SPARGE_OK;
  if (mask == nullptr || kv_idx == nullptr || kv_cnt == nullptr) return SPARGE_EINVAL;
  if ((reinterpret_cast<uintptr_t>(kv_idx) & 3u) || (reinterpret_cast<uintptr_t>(kv_cnt) & 3u))
    return SPARGE_EINVAL;
  DeviceScope dev;
  if ((st = dev.enter(kv_idx)) != SPARGE_OK) return st;
  return from_cuda(launch_mask_compact(*p, mask, kv_idx, kv_cnt, stream));
}

sparge_status_t sparge_attn_fwd(const sparge_params_t* p, const void* q, const void* k,
                                const void* v, const int32_t* kv_idx, const int32_t* kv_cnt,
                                void* o, void* ws, size_t ws_bytes, sparge_stats_t* stats,
                                cudaStream_t stream) {
  sparge_status_t st = check_params(p);
  if (st != SPARGE_OK) return st;
  if (empty_problem(p)) return SPARGE_OK;
  if (q == nullptr || k == nullptr || v == nullptr || kv_idx == nullptr || kv_cnt == nullptr ||
      o == nullptr || ws == nullptr)
    return SPARGE_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) || (reinterpret_cast<uintptr_t>(kv_idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(kv_cnt) & 3u) || (reinterpret_cast<uintptr_t>(stats) & 7u))
    return SPARGE_EINVAL;
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.total) return SPARGE_EWORKSPACE;
  DeviceScope dev;
  if ((st = dev.enter(q)) != SPARGE_OK) return st;
  AttnPtrs x{};
  x.q = p->qk_int8 ? static_cast<const void*>(ws_ptr<int8_t>(ws, L.q_codes)) : q;
  x.k = p->qk_int8 ? static_cast<const void*>(ws_ptr<int8_t>(ws, L.k_codes)) : k;
  if (p->io_dtype == SPARGE_BF16) {
    x.v16 = ws_ptr<void>(ws, L.v16);
    x.v = x.v16;
    x.v_io = v;
  } else {
    x.v16 = nullptr;
    x.v = v;
    x.v_io = v;
  }
  x.dq = p->qk_int8 ? ws_ptr<float>(ws, L.dq) : nullptr;
  x.dk = p->qk_int8 ? ws_ptr<float>(ws, L.dk) : nullptr;
  x.kv_idx = kv_idx;
  x.kv_cnt = kv_cnt;
  x.o = o;
  x.status = ws_ptr<int32_t>(ws, L.status);
  x.stats = stats;
  return from_cuda(launch_attention(*p, x, stream));
}

sparge_status_t sparge_device_status(void* ws, cudaStream_t stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPARGE_EINVAL;
  DeviceScope dev;
  sparge_status_t st = dev.enter(ws);
  if (st != SPARGE_OK) return st;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SPARGE_ECUDA;
  int32_t h = 0;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SPARGE_ECUDA;
  if (h != 0 && cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return SPARGE_ECUDA;
  return static_cast<sparge_status_t>(h);
}

const char* sparge_status_string(sparge_status_t s) {
  switch (s) {
    case SPARGE_OK: return "ok";
    case SPARGE_EINVAL: return "invalid argument";
    case SPARGE_EUNSUPPORTED: return "unsupported configuration";
    case SPARGE_ECUDA: return "CUDA runtime error";
    case SPARGE_ETIMEOUT: return "device wait timed out";
    case SPARGE_EWORKSPACE: return "workspace too small";
    case SPARGE_ERANGE: return "value outside the fp16 range was saturated";
  }
  return "unknown status";
}

}  // extern "C"
