// Stage 1 of SpargeAttn: the sparse-block predictor (paper review page,
// section 三, Eq. 4-9 and Algorithm 1 steps 2-5).
//
//   pool_warp_kernel<.., 0>  one pass over Q and K (HBM bound), one warp per
//                   block: the mean token (Eq. 4, 5) and the self-similarity
//                   CosSim (Eq. 6, read as the mean of the block's token cosine
//                   matrix), via mean_{a,b} xh_a.xh_b = |sum_a xh_a|^2 / n^2.
//                   With INT8 it also quantises Q per block (Algorithm 1 step 2).
//   kbar_kernel     per-head mean of K from the block means (K smoothing).
//   pool_warp_kernel<.., 1>  per-block INT8 of K - kbar (second pass over K).
//   select_kernel   per query block: S_hat = scale q_i k^T with -inf columns
//                   (Eq. 7), row softmax, TopCdf(tau) (Eq. 8) by an exact
//                   value-threshold bisection, the fix-block rule (Eq. 9), and
//                   the ascending per-tile skip list.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cfloat>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "sparge_internal.h"

namespace sparge {
namespace {

constexpr int kPoolThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& raw, float (&x)[8], bool bf16) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (bf16) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 f = __half22float2(h);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

// code = rint(x * inv), inv = 127 / absmax of the block, clamped to +-127
__device__ __forceinline__ int8_t quant1(float x, float inv) {
  float v = rintf(__fmul_rn(x, inv));
  v = fminf(127.f, fmaxf(-127.f, v));
  return static_cast<int8_t>(v);
}

__device__ __forceinline__ uint2 pack_codes(const float (&x)[8], float inv) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) lo |= (uint32_t)(uint8_t)quant1(x[e], inv) << (8 * e);
#pragma unroll
  for (int e = 0; e < 4; ++e) hi |= (uint32_t)(uint8_t)quant1(x[4 + e], inv) << (8 * e);
  return make_uint2(lo, hi);
}

struct PoolArgs {
  const void* q;
  const void* k;
  int32_t N, bq, bk, Tm, Tn;
  int64_t nQblocks;  // B*Hq*Tm: Q blocks come first in the pooling pass
  int64_t nblocks;   // blocks this pass visits
  float* q_mean;
  float* k_mean;
  float* s_q;
  float* s_k;
  int8_t* q_codes;   // nullable: quantise Q in the pooling pass
  float* dq;
  const float* kbar; // INT8 pass over K - kbar
  int8_t* k_codes;
  float* dk;
  int32_t* status;
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One warp per block, no shared memory and no CTA barrier: lane (ro, c) owns
// the 16-byte chunk c of rows ro, ro + RPW, ...  Row norms reduce over the CH
// lanes of a row, column sums over the RPW row groups at the end.
//   KIND 0  pooling pass over Q blocks then K blocks: mean token, CosSim by
//           |sum xhat|^2 / n^2, and with q_codes the INT8 codes of Q.
//   KIND 1  INT8 pass over K blocks: codes of K - kbar and their scales.
// The codes are a second, L2-resident read of the block once its absmax is
// known: code = rint(x * (127 / absmax)), clamped to +-127.
template <int D, bool BF16, int KIND>
__global__ void __launch_bounds__(256) pool_warp_kernel(PoolArgs a) {
  constexpr int CH = D * 2 / 16;          // lanes per row
  constexpr int RPW = 32 / CH;            // rows per warp pass
  constexpr int UNROLL = 4;
  const int lane = threadIdx.x & 31;
  const int64_t id0 = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (id0 >= a.nblocks) return;
  int64_t id = id0;
  const bool isQ = KIND == 0 && id < a.nQblocks;
  if (KIND == 0 && !isQ) id -= a.nQblocks;
  const int T = isQ ? a.Tm : a.Tn;
  const int BLK = isQ ? a.bq : a.bk;
  const int64_t bh = id / T;
  const int blk = int(id % T);
  const int rows = min(BLK, a.N - blk * BLK);
  const uint16_t* src = static_cast<const uint16_t*>(isQ ? a.q : a.k) +
                        (bh * a.N + int64_t(blk) * BLK) * D;
  const int c = lane % CH, ro = lane / CH;

  float kb[8];
  if (KIND == 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) kb[e] = a.kbar[bh * D + c * 8 + e];
  }
  float sx[8], su[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sx[e] = su[e] = 0.f;
  float amax = 0.f;
  for (int r0 = ro; r0 < BLK; r0 += RPW * UNROLL) {
    uint4 raw[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int r = r0 + u * RPW;
      raw[u] = r < rows ? ld_stream(src + int64_t(r) * D + c * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const bool valid = r0 + u * RPW < rows;
      float x[8];
      unpack8(raw[u], x, BF16);
      if (KIND == 0) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int o = CH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          sx[e] += x[e];
          su[e] = fmaf(x[e], inv, su[e]);
          amax = fmaxf(amax, fabsf(x[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (valid) amax = fmaxf(amax, fabsf(__fsub_rn(x[e], kb[e])));
      }
    }
  }
  if (KIND == 0) {
    // column sums over the RPW row groups
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sx[e] += __shfl_xor_sync(0xffffffffu, sx[e], o);
        su[e] += __shfl_xor_sync(0xffffffffu, su[e], o);
      }
    float uu = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) uu = fmaf(su[e], su[e], uu);
#pragma unroll
    for (int o = CH / 2; o > 0; o >>= 1) uu += __shfl_xor_sync(0xffffffffu, uu, o);
    float* mean = isQ ? a.q_mean : a.k_mean;
    if (lane < CH) {
      const float n = float(rows);
      float4* dst = reinterpret_cast<float4*>(mean + (bh * T + blk) * D + c * 8);
      dst[0] = make_float4(sx[0] / n, sx[1] / n, sx[2] / n, sx[3] / n);
      dst[1] = make_float4(sx[4] / n, sx[5] / n, sx[6] / n, sx[7] / n);
    }
    if (lane == 0) (isQ ? a.s_q : a.s_k)[bh * T + blk] = uu / (float(rows) * float(rows));
  }
  const bool quantise = KIND == 1 || (isQ && a.q_codes != nullptr);
  if (!quantise) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float delta = amax / 127.0f;
  const float inv = amax > 0.f ? 127.0f / amax : 0.f;
  if (lane == 0) (KIND == 1 ? a.dk : a.dq)[bh * T + blk] = delta;
  int8_t* codes = (KIND == 1 ? a.k_codes : a.q_codes) + (bh * a.N + int64_t(blk) * BLK) * D;
  for (int r0 = ro; r0 < rows; r0 += RPW * UNROLL) {
    uint4 raw[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int r = r0 + u * RPW;
      raw[u] = r < rows ? *reinterpret_cast<const uint4*>(src + int64_t(r) * D + c * 8)
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int r = r0 + u * RPW;
      if (r < rows) {
        float x[8];
        unpack8(raw[u], x, BF16);
        if (KIND == 1) {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], kb[e]);
        }
        *reinterpret_cast<uint2*>(codes + int64_t(r) * D + c * 8) = pack_codes(x, inv);
      }
    }
  }
}

// kbar[bh, :] = (sum_j n_j * k_mean[bh, j, :]) / N, a fixed-order two-level sum
template <int D>
__global__ void __launch_bounds__(1024) kbar_kernel(const float* k_mean, float* kbar, int32_t N,
                                                    int32_t bk, int32_t Tn) {
  constexpr int G = 1024 / D;
  __shared__ float part[G][D];
  const int64_t bh = blockIdx.x;
  const int g = threadIdx.x / D, col = threadIdx.x % D;
  float acc = 0.f;
  for (int j = g; j < Tn; j += G) {
    const int n = min(bk, N - j * bk);
    acc = fmaf(k_mean[(bh * Tn + j) * D + col], float(n), acc);
  }
  part[g][col] = acc;
  __syncthreads();
  if (g == 0) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < G; ++i) s += part[i][col];
    kbar[bh * D + col] = s / float(N);
  }
}

// ------------------------------------------------------------------ select
constexpr int kSelRows = 8;   // query blocks per CTA (one warp each)
constexpr int kSelCols = 256; // key blocks scored per pass (one thread each)
constexpr int kKPad = 36;     // padded row of a staged 32-float k chunk

struct SelectArgs {
  const float* q_mean;
  const float* k_mean;
  const float* s_q;
  const float* s_k;
  uint8_t* mask;
  int32_t* kv_idx;
  int32_t* kv_cnt;
  int32_t Hq, Hkv, N, bq, bk, Tm, Tn, causal;
  float tau, theta, scale;
};

__device__ __forceinline__ int visible_cols(int i, int N, int bq, int bk, int Tn, int causal) {
  if (!causal) return Tn;
  const int last_row = min(N, (i + 1) * bq) - 1;
  return min(Tn, last_row / bk + 1);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D>
__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                        // [kSelRows][D]
  float* ks = qs + kSelRows * D;           // [kSelCols][kKPad]
  float* shat = ks + kSelCols * kKPad;     // [kSelRows][Tn]

  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kSelRows;
  const int g = a.Hq / a.Hkv;
  const int64_t bh = int64_t(b) * a.Hq + h;
  const int64_t kbh = int64_t(b) * a.Hkv + h / g;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int i_last = min(a.Tm, i0 + kSelRows) - 1;
  const int jcount = visible_cols(i_last, a.N, a.bq, a.bk, a.Tn, a.causal);

  for (int idx = tid; idx < kSelRows * D; idx += 256) {
    const int r = idx / D, e = idx % D;
    qs[idx] = (i0 + r < a.Tm) ? a.q_mean[(bh * a.Tm + i0 + r) * D + e] : 0.f;
  }
  // ---- S_hat rows i0..i0+7 against every visible key block (Eq. 7, before masking)
  for (int jt = 0; jt * kSelCols < jcount; ++jt) {
    float acc[kSelRows];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
    for (int ec = 0; ec < D; ec += 32) {
      __syncthreads();
      for (int idx = tid; idx < kSelCols * 8; idx += 256) {
        const int jl = idx >> 3, f4 = idx & 7, j = jt * kSelCols + jl;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < jcount)
          v = *reinterpret_cast<const float4*>(a.k_mean + (kbh * a.Tn + j) * D + ec + f4 * 4);
        *reinterpret_cast<float4*>(ks + jl * kKPad + f4 * 4) = v;
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(ks + tid * kKPad + e);
#pragma unroll
        for (int r = 0; r < kSelRows; ++r) {
          const float4 qv = *reinterpret_cast<const float4*>(qs + r * D + ec + e);
          acc[r] = fmaf(qv.x, kv.x, acc[r]);
          acc[r] = fmaf(qv.y, kv.y, acc[r]);
          acc[r] = fmaf(qv.z, kv.z, acc[r]);
          acc[r] = fmaf(qv.w, kv.w, acc[r]);
        }
      }
    }
    const int j = jt * kSelCols + tid;
    if (j < jcount) {
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) shat[r * a.Tn + j] = acc[r] * a.scale;
    }
  }
  __syncthreads();

  // ---- one warp per query block: softmax, TopCdf, fix rule, compaction
  const int i = i0 + w;
  if (i >= a.Tm) return;
  float* row = shat + w * a.Tn;
  const int nvis = visible_cols(i, a.N, a.bq, a.bk, a.Tn, a.causal);
  const bool fix_row = a.s_q[bh * a.Tm + i] < a.theta;
  const float* sk = a.s_k + kbh * a.Tn;

  float mx = -INFINITY;
  for (int j = lane; j < nvis; j += 32) {
    const float v = sk[j] >= a.theta ? row[j] : -INFINITY;
    row[j] = v;
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  // unnormalised softmax weights; -1 marks a -inf entry
  float tot = 0.f;
  for (int j = lane; j < nvis; j += 32) {
    const float v = row[j];
    const float e = (v == -INFINITY) ? -1.f : expf(v - mx);
    row[j] = e;
    tot += fmaxf(e, 0.f);
  }
  tot = warp_sum(tot);
  __syncwarp();
  float t_star = 0.f;  // keep e >= t_star (t_star = 0 keeps every finite entry)
  if (a.tau < 1.0f) {
    // largest t with sum_{e >= t} e >= tau * total: an exact value of the row
    const float target = a.tau * tot;
    uint32_t lo = 0u, hi = 0x3F800001u;  // f(lo) >= target, f(hi) = 0 < target
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      const float t = __uint_as_float(mid);
      float f = 0.f;
      for (int j = lane; j < nvis; j += 32) {
        const float e = row[j];
        f += (e >= t) ? e : 0.f;
      }
      f = warp_sum(f);
      if (f >= target)
        lo = mid;
      else
        hi = mid;
    }
    t_star = __uint_as_float(lo);
  }
  const int64_t out = (bh * a.Tm + i) * a.Tn;
  int cnt = 0;
  for (int jb = 0; jb < a.Tn; jb += 32) {
    const int j = jb + lane;
    bool keep = false;
    if (j < nvis) {
      const float e = row[j];
      keep = (e >= 0.f && e >= t_star) || fix_row || sk[j] < a.theta;
    }
    if (j < a.Tn) a.mask[out + j] = keep ? 1 : 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (keep) a.kv_idx[out + cnt + __popc(bal & ((1u << lane) - 1u))] = j;
    cnt += __popc(bal);
  }
  if (lane == 0) a.kv_cnt[bh * a.Tm + i] = cnt;
}

__global__ void compact_kernel(const uint8_t* mask, int32_t* kv_idx, int32_t* kv_cnt,
                               int64_t rows, int32_t Tn) {
  const int64_t r = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint8_t* m = mask + r * Tn;
  int cnt = 0;
  for (int jb = 0; jb < Tn; jb += 32) {
    const int j = jb + lane;
    const bool keep = j < Tn && m[j] != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (keep) kv_idx[r * Tn + cnt + __popc(bal & ((1u << lane) - 1u))] = j;
    cnt += __popc(bal);
  }
  if (lane == 0) kv_cnt[r] = cnt;
}

template <int D, bool BF16>
cudaError_t predict_impl(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
  PoolArgs pa{};
  pa.q = x.q;
  pa.k = x.k;
  pa.N = p.N;
  pa.bq = p.bq;
  pa.bk = p.bk;
  pa.Tm = int32_t(Tm);
  pa.Tn = int32_t(Tn);
  pa.nQblocks = int64_t(p.B) * p.Hq * Tm;
  pa.nblocks = pa.nQblocks + int64_t(p.B) * p.Hkv * Tn;
  pa.q_mean = x.q_mean;
  pa.k_mean = x.k_mean;
  pa.s_q = x.s_q;
  pa.s_k = x.s_k;
  pa.q_codes = x.q_codes;
  pa.dq = x.dq;
  pa.status = x.status;
  cudaError_t e;
  const int64_t warps_per_cta = kPoolThreads / 32;
  pool_warp_kernel<D, BF16, 0>
      <<<unsigned(cdiv(pa.nblocks, warps_per_cta)), kPoolThreads, 0, s>>>(pa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (x.k_codes != nullptr) {
    kbar_kernel<D><<<unsigned(int64_t(p.B) * p.Hkv), 1024, 0, s>>>(x.k_mean, x.kbar, p.N, p.bk,
                                                                   int32_t(Tn));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    PoolArgs qa = pa;
    qa.nblocks = int64_t(p.B) * p.Hkv * Tn;
    qa.nQblocks = 0;
    qa.kbar = x.kbar;
    qa.k_codes = x.k_codes;
    qa.dk = x.dk;
    pool_warp_kernel<D, BF16, 1>
        <<<unsigned(cdiv(qa.nblocks, warps_per_cta)), kPoolThreads, 0, s>>>(qa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  SelectArgs sa{};
  sa.q_mean = x.q_mean;
  sa.k_mean = x.k_mean;
  sa.s_q = x.s_q;
  sa.s_k = x.s_k;
  sa.mask = x.mask;
  sa.kv_idx = x.kv_idx;
  sa.kv_cnt = x.kv_cnt;
  sa.Hq = p.Hq;
  sa.Hkv = p.Hkv;
  sa.N = p.N;
  sa.bq = p.bq;
  sa.bk = p.bk;
  sa.Tm = int32_t(Tm);
  sa.Tn = int32_t(Tn);
  sa.causal = p.causal;
  sa.tau = p.tau;
  sa.theta = p.theta;
  sa.scale = p.scale;
  const size_t smem = sizeof(float) * (kSelRows * D + kSelCols * kKPad + kSelRows * Tn);
  e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem));
  if (e != cudaSuccess) return e;
  dim3 sgrid{unsigned(cdiv(Tm, kSelRows)), unsigned(p.Hq), unsigned(p.B)};
  select_kernel<D><<<sgrid, 256, smem, s>>>(sa);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_predict(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  const bool bf16 = p.io_dtype == SPARGE_BF16;
  if (p.d == 128) return bf16 ? predict_impl<128, true>(p, x, s) : predict_impl<128, false>(p, x, s);
  if (p.d == 64) return bf16 ? predict_impl<64, true>(p, x, s) : predict_impl<64, false>(p, x, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_mask_compact(const sparge_params_t& p, const uint8_t* mask, int32_t* kv_idx,
                                int32_t* kv_cnt, cudaStream_t s) {
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
  const int64_t rows = int64_t(p.B) * p.Hq * Tm;
  compact_kernel<<<unsigned(cdiv(rows, 8)), 256, 0, s>>>(mask, kv_idx, kv_cnt, rows,
                                                          int32_t(Tn));
  return cudaGetLastError();
}

}  // namespace sparge
