// Internal declarations shared by the host entry points and the kernels:
// workspace carving and the launchers of each kernel family.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sparge.h"

namespace sparge {

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Offsets (bytes) of every region of the caller's workspace.
struct WsLayout {
  size_t status;    // int32 status word (kernels OR/CAS error codes in)
  size_t q_mean;    // [B, Hq, Tm, d] f32
  size_t k_mean;    // [B, Hkv, Tn, d] f32
  size_t s_q;       // [B, Hq, Tm] f32
  size_t s_k;       // [B, Hkv, Tn] f32
  size_t v16;       // [B, Hkv, N, d] f16 (bf16 I/O only), else npos
  size_t q_codes;   // [B, Hq, N, d] int8 (qk_int8), else npos
  size_t k_codes;   // [B, Hkv, N, d] int8
  size_t dq;        // [B, Hq, Tm] f32
  size_t dk;        // [B, Hkv, Tn] f32
  size_t kbar;      // [B, Hkv, d] f32
  size_t k_sum64;   // [B, Hkv, Tn, d] f64 column sums of every K block
  size_t total;
  static constexpr size_t npos = ~size_t(0);
};

inline WsLayout ws_layout(const sparge_params_t& p) {
  WsLayout w{};
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  w.status = take(256);
  w.q_mean = take(size_t(p.B) * p.Hq * Tm * p.d * 4);
  w.k_mean = take(size_t(p.B) * p.Hkv * Tn * p.d * 4);
  w.s_q = take(size_t(p.B) * p.Hq * Tm * 4);
  w.s_k = take(size_t(p.B) * p.Hkv * Tn * 4);
  w.v16 = p.io_dtype == SPARGE_BF16 ? take(size_t(p.B) * p.Hkv * p.N * p.d * 2) : WsLayout::npos;
  if (p.qk_int8) {
    w.q_codes = take(size_t(p.B) * p.Hq * p.N * p.d);
    w.k_codes = take(size_t(p.B) * p.Hkv * p.N * p.d);
    w.dq = take(size_t(p.B) * p.Hq * Tm * 4);
    w.dk = take(size_t(p.B) * p.Hkv * Tn * 4);
    w.kbar = take(size_t(p.B) * p.Hkv * p.d * 4);
    w.k_sum64 = take(size_t(p.B) * p.Hkv * Tn * p.d * 8);
  } else {
    w.q_codes = w.k_codes = w.dq = w.dk = w.kbar = w.k_sum64 = WsLayout::npos;
  }
  w.total = off;
  return w;
}

template <typename T>
inline T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Host validation of a parameter set shared by every entry point that takes
// one: SPARGE_OK, SPARGE_EINVAL or SPARGE_EUNSUPPORTED (sparge_api.cu).
sparge_status_t check_params(const sparge_params_t* p);

// Makes the device that owns a pointer current for one entry point and puts
// the caller's current device back when it leaves scope.
class DeviceScope {
 public:
  DeviceScope() = default;
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  ~DeviceScope() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }
  // SPARGE_EINVAL when ptr is not device (or managed) memory.
  sparge_status_t enter(const void* ptr) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
      cudaGetLastError();
      return SPARGE_EINVAL;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return SPARGE_EINVAL;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return SPARGE_ECUDA;
    if (cur != a.device) {
      if (cudaSetDevice(a.device) != cudaSuccess) return SPARGE_ECUDA;
      prev_ = cur;
    }
    device_ = a.device;
    return SPARGE_OK;
  }
  int device() const { return device_; }

 private:
  int prev_ = -1;
  int device_ = -1;
};

// ------------------------------------------------------------- predict.cu
struct PredictPtrs {
  const void* q;
  const void* k;
  float* q_mean;
  float* k_mean;
  float* s_q;
  float* s_k;
  int8_t* q_codes;  // nullable
  int8_t* k_codes;  // nullable
  float* dq;
  float* dk;
  float* kbar;
  double* ksum64;
  uint8_t* mask;
  int32_t* kv_idx;
  int32_t* kv_cnt;
  int32_t* status;  // device status word (timeouts of the bounded waits)
};
// pooling, self-similarity and INT8 codes (writes the workspace regions) ...
cudaError_t launch_predict_pool(const sparge_params_t& p, const PredictPtrs& ptrs, cudaStream_t s);
// ... then S_hat, TopCdf, the fix rule and the skip list from them
cudaError_t launch_predict_select(const sparge_params_t& p, const PredictPtrs& ptrs,
                                  cudaStream_t s);
cudaError_t launch_predict(const sparge_params_t& p, const PredictPtrs& ptrs, cudaStream_t s);
cudaError_t launch_mask_compact(const sparge_params_t& p, const uint8_t* mask, int32_t* kv_idx,
                                int32_t* kv_cnt, cudaStream_t s);

// ------------------------------------------------------------- permute.cu
size_t hilbert_ws_bytes(int32_t T, int32_t Hg, int32_t Wg);
cudaError_t launch_hilbert_index(int32_t N, int32_t prefix_len, int32_t T, int32_t Hg,
                                 int32_t Wg, int32_t* perm, void* ws, cudaStream_t s);
cudaError_t launch_permute_rows(const void* x, void* y, int64_t BH, int32_t N, int32_t row_bytes,
                                const int32_t* perm, bool inverse, cudaStream_t s);

// ------------------------------------------------------------- attn_sm100.cu
struct AttnPtrs {
  const void* q;        // io dtype, or int8 codes with qk_int8
  const void* k;        // io dtype, or int8 codes
  const void* v;        // io dtype (f16) or the f16 copy in ws
  const void* v_io;     // caller's V (bf16 when a conversion is needed)
  void* v16;            // conversion target, or nullptr when V is already f16
  const float* dq;      // qk_int8 block scales
  const float* dk;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  void* o;
  int32_t* status;
  sparge_stats_t* stats;
};
// Returns cudaErrorNotSupported when no TMA descriptor could be built.
cudaError_t launch_attention(const sparge_params_t& p, const AttnPtrs& ptrs, cudaStream_t s);

}  // namespace sparge
