// Stage 1 of SpargeAttn: the sparse-block predictor (paper review page,
// section 三, Eq. 4-9 and Algorithm 1 steps 2-5).
//
//   pool_kernel<.., 0>  one pass over Q (and, without INT8, K; HBM bound),
//                   one warp per slab of 32 rows (64 at d = 64) held in
//                   registers: the mean token (Eq. 4, 5) and the
//                   self-similarity CosSim (Eq. 6, read as the mean of the
//                   block's token cosine matrix), via
//                   mean_{a,b} xh_a.xh_b = |sum_a xh_a|^2 / n^2.  With INT8 it
//                   also quantises Q per block (Algorithm 1 step 2).
//   pool_kernel<.., 2>  with INT8, the pooling pass over K alone, which also
//                   writes each K block's float64 column sums;
//   kbar_kernel     per-head mean of K from them (K smoothing);
//   pool_kernel<.., 1>  per-block INT8 of K - kbar (second pass over K).
//   select_kernel   per query block: S_hat = scale q_i k^T with -inf columns
//                   (Eq. 7), row softmax, TopCdf(tau) (Eq. 8) by an exact
//                   radix select of the threshold value, the fix-block rule
//                   (Eq. 9), and the ascending per-tile skip list.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cfloat>
#include <climits>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "sparge_internal.h"

namespace sparge {
namespace {

constexpr int kPoolBQ = 128;       // query block rows (the only b_q the library accepts)
constexpr int kPoolBK = 64;        // key block rows
constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
// Warps of a pooling CTA: at least four, and all the slabs of one query block.
constexpr int pool_warps(int slab) { return kPoolBQ / slab > 4 ? kPoolBQ / slab : 4; }
// CTAs per SM the register budget is set for: four 4-warp CTAs (128 registers;
// a 32-row slab's rows take 64 of them), or two 8-warp CTAs.  (16-row slabs,
// eight warps to a query block, ran the 128K pooling stage 35% slower than
// 32-row slabs: the per-slab reductions and barriers cost more than the extra
// warps hide.)
constexpr int pool_min_blocks(int slab) { return pool_warps(slab) == 4 ? 4 : 2; }

// n / d for 0 <= n < 2^31 and a divisor 1 <= d < 2^31 known when the kernel
// is launched, by a multiply (Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (umulhi(n, m) + n) >> l; the sum
// stays below 2^32 because n < 2^31.
struct FastDiv {
  uint32_t mul, shr;
  static FastDiv make(uint32_t d) {
    uint32_t l = 0;
    while ((uint64_t(1) << l) < d) ++l;
    const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1;
    return FastDiv{uint32_t(m), l};
  }
};
__device__ __forceinline__ int fast_div(int n, uint32_t mul, uint32_t shr) {
  return int((__umulhi(uint32_t(n), mul) + uint32_t(n)) >> shr);
}

struct PoolArgs {
  const void* q;
  const void* k;
  int32_t N, bq, bk, Tm, Tn;
  uint32_t tm_mul, tm_shr, tn_mul, tn_shr;  // n / Tm and n / Tn by multiply (FastDiv)
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
  double* ksum64;    // KIND 2: [B, Hkv, Tn, D] float64 column sums of the K blocks
  int32_t* status;
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16 bytes global -> shared, cached in L2 only; completed by cp_async_wait.
// bytes is 16, or 0 to fill the 16 shared bytes with zeros and read nothing.
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Same bits, but opaque to the compiler: keeps it from holding every row's
// unpacked floats live between two passes over the registers (it would
// otherwise reuse the first unpacking and spill).
__device__ __forceinline__ uint4 opaque(uint4 v) {
  asm volatile("" : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w));
  return v;
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// The two 16-bit values of w as a packed fp32 pair (exact).
template <bool BF16>
__device__ __forceinline__ uint64_t widen2(uint32_t w) {
  if (BF16) return pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  return pack2(f.x, f.y);
}

// Per-half running max of |x| on packed 16-bit values: max.xorsign.abs keeps
// the larger magnitude (its sign bit is dropped at the end).  Exact.
template <bool BF16>
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {
  uint32_t r;
  if (BF16)
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
  else
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
  return r;
}

// Per-half max and min of packed 16-bit values (exact).
template <bool BF16>
__device__ __forceinline__ uint32_t max2_16(uint32_t a, uint32_t b) {
  uint32_t r;
  if (BF16)
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else
    asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <bool BF16>
__device__ __forceinline__ uint32_t min2_16(uint32_t a, uint32_t b) {
  uint32_t r;
  if (BF16)
    asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else
    asm("min.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <bool BF16>
__device__ __forceinline__ float absmax2_value(uint32_t acc) {
  const uint32_t m = acc & 0x7FFF7FFFu;
  if (BF16) return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&m));
  return fmaxf(f.x, f.y);
}

// rint(x / delta) of eight values by the IEEE division itself, as the bits
// of q + 1.5 * 2^23 (the code is their low byte).  Out of line: it runs only
// for a subnormal delta, and inlined into every unrolled row of the pooling
// kernel it would make the kernel's code too large for the instruction cache.
__device__ __noinline__ uint2 codes8_exact(float x0, float x1, float x2, float x3, float x4,
                                           float x5, float x6, float x7, float delta) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float x[8] = {x0, x1, x2, x3, x4, x5, x6, x7};
  uint32_t bits[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) bits[i] = __float_as_uint(__fadd_rn(__fdiv_rn(x[i], delta), kMagic));
  const uint32_t lo = __byte_perm(__byte_perm(bits[0], bits[1], 0x0040),
                                  __byte_perm(bits[2], bits[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(bits[4], bits[5], 0x0040),
                                  __byte_perm(bits[6], bits[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// Eight INT8 codes rint(x / delta): round half to even of the IEEE float32
// quotient.  The quotient comes from the reciprocal y = RN(1/delta) by
// Markstein's final correction step for division with a fused multiply-add:
// q0 = RN(x y), r = RN(x - q0 delta), q = RN(q0 + r y), which is the correctly
// rounded x / delta (it is the last step of FMA-based IEEE division; checked
// here against exact rational arithmetic on bf16 and float32 inputs, on
// quotients at and next to half-integers, and by the bit-exact GPU tests).
// Then q + 1.5 * 2^23 rounds q to the nearest integer, ties to even, exactly
// (|q| < 2^22), and the code is the low byte of that sum's bits, two's
// complement included.  Every step is an explicit .rn instruction on packed
// pairs, so nothing is fused or reordered.  A subnormal delta, whose
// reciprocal overflows, takes the IEEE division instead.
__device__ __forceinline__ uint2 codes8(const uint64_t (&x2)[4], float inv, float delta,
                                        bool exact_only) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  if (exact_only) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack2(x2[i], v[2 * i], v[2 * i + 1]);
    return codes8_exact(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], delta);
  }
  const uint64_t inv2 = pack2(inv, inv), nd2 = pack2(-delta, -delta), mg2 = pack2(kMagic, kMagic);
  uint32_t bits[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t q0 = mul2(x2[i], inv2);
    const uint64_t r = fma2(q0, nd2, x2[i]);    // x - q0 delta
    const uint64_t q = fma2(r, inv2, q0);       // q0 + r y
    float r0, r1;
    unpack2(add2(q, mg2), r0, r1);
    bits[2 * i] = __float_as_uint(r0);
    bits[2 * i + 1] = __float_as_uint(r1);
  }
  const uint32_t lo = __byte_perm(__byte_perm(bits[0], bits[1], 0x0040),
                                  __byte_perm(bits[2], bits[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(bits[4], bits[5], 0x0040),
                                  __byte_perm(bits[6], bits[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// x * 2^-896 as a float64, built from the float32 bits of x (the fp64
// conversion unit runs at a quarter of the integer rate): the exponent field
// is kept as it stands, so bias 127 reads as bias 1023, and the significand
// moves down three places into the high word.  A normal x becomes the normal
// float64 x * 2^-896 and a float32 subnormal 0.f * 2^-126 (a bf16 below
// 2^-126) the float64 subnormal 0.f * 2^-1022, the same scaling.  Exact for
// every finite float32 whose low three significand bits are zero, which holds
// for every widened bf16 or f16 value.  Sums taken in this domain round
// exactly as the unscaled float64 sums would: every partial sum below 2^-126
// is a multiple of 2^-133 with at most seven significant bits, exact in both.
constexpr double kF64Unscale = 0x1p896;
__device__ __forceinline__ double f64_scaled(float x) {
  // arithmetic shift: the sign fills bits 31..28, the mask keeps bit 31
  const uint32_t hi = uint32_t(int32_t(__float_as_uint(x)) >> 3) & 0x8FFFFFFFu;
  return __hiloint2double(int(hi), 0);
}

// One warp per SLAB-row slab of a block, held in registers while the block
// is processed, so every byte of Q and K is read from HBM exactly once per
// pass.  A CTA of four warps takes units of four slabs (one Q block or two K
// blocks); the Q pass and the K code pass are persistent, taking units in a
// grid-stride loop, and each warp copies its slab of the next unit into its
// shared-memory buffer (cp.async; rows past a ragged end are zero-filled)
// while it works on the current one, so loads stay in flight all the time.
// Lane (ro, c) owns the 16-byte chunk c of rows ro, ro + RPW, ...  Arithmetic
// runs on packed fp32 pairs in two sweeps over the registers: the first takes
// the squared row norms, the column sums of x and the exact |x| max; the
// second, once the block's absmax is known, the column sums of x / |x_row|
// and the INT8 codes.  The row norms are reduced over the CH lanes of each row
// by a transposing butterfly (each step halves the rows a lane carries) and
// the inverse norms broadcast back.  The G = block rows / SLAB warps of one
// block are adjacent in the CTA and combine their partial sums and absmax
// through shared memory (named barriers), always in slab order, so the result
// does not depend on scheduling.
//   KIND 0  pooling pass over Q blocks then K blocks: mean token, CosSim by
//           |sum xhat|^2 / n^2, and with q_codes the INT8 codes of Q.
//   KIND 1  INT8 pass over K blocks, last block first (the blocks pooled last
//           are still in L2): codes of K - kbar and their scales.
//   KIND 2  pooling pass over K blocks that also writes every block's column
//           sums in float64 (exact for 16-bit inputs), from which kbar is the
//           float64 mean rounded once to float32.
template <int D, bool BF16, int KIND, int SLAB>
__global__ void __launch_bounds__(32 * pool_warps(SLAB), pool_min_blocks(SLAB))
    pool_kernel(PoolArgs a) {
  constexpr bool POOL = KIND != 1;
  constexpr bool SUM64 = KIND == 2;
  // The Q pass and the K code pass are persistent and stage the next unit in
  // shared memory; the K pooling pass takes one unit per CTA and loads
  // straight into registers (its float64 sums leave no registers for the
  // loop's state).
  constexpr bool PERSIST = KIND != 2;
  constexpr int CH = D * 2 / 16;  // lanes per row
  constexpr int RPW = 32 / CH;    // rows per warp-wide load
  constexpr int NR = SLAB / RPW;  // rows per lane
  // after the butterfly a lane holds the norms of R rows, and each row's norm
  // is held by SPREAD adjacent lanes
  constexpr int R = NR >= CH ? NR / CH : 1;
  constexpr int SPREAD = NR >= CH ? 1 : CH / NR;
  constexpr int WARPS = pool_warps(SLAB);
  constexpr int GQ = kPoolBQ / SLAB, GK = kPoolBK / SLAB;
  static_assert(WARPS % GQ == 0 && GQ % GK == 0, "groups must tile the CTA");
  static_assert(NR % CH == 0 || CH % NR == 0, "butterfly needs NR and CH nested");
  __shared__ __align__(16) float part[WARPS][2 * D];
  __shared__ float pmax[WARPS];
  __shared__ __align__(16) double part64[SUM64 ? WARPS : 1][SUM64 ? D : 1];
  __shared__ __align__(16) uint4 stage[PERSIST ? WARPS : 1][PERSIST ? NR : 1][32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane % CH, ro = lane / CH;
  // this lane's eight columns of a warp's partial sums, as 16-byte words
  auto part8 = [&](int w, int off) { return reinterpret_cast<float4*>(&part[w][off + c * 8]); };
  auto part64_8 = [&](int w) { return reinterpret_cast<double2*>(&part64[w][c * 8]); };
  const int64_t nQw = a.nQblocks * GQ;
  const int64_t n_units = (nQw + (a.nblocks - a.nQblocks) * GK + WARPS - 1) / WARPS;
  // the slab that this warp takes in unit u: Q blocks first, then K blocks
  // (KIND 1 walks its K blocks last first); whole groups of G warps are
  // either inside or past the end
  struct Slab {
    bool valid, isQ;
    int64_t bh, row0;
    int blk, sub, rows, srows;
  };
  // (32-bit indices: the library refuses parameter sets with 2^31 tiles or
  // more, and the group sizes G are powers of two)
  auto slab_of = [&](int64_t u) {
    Slab sl;
    const int64_t gw64 = u * WARPS + warp;
    const int gw = gw64 < INT32_MAX ? int(gw64) : INT32_MAX;
    const int nqw = int(nQw);
    sl.isQ = KIND == 0 && gw < nqw;
    const int lg = sl.isQ ? ilog2(GQ) : ilog2(GK);
    const int rel = sl.isQ ? gw : gw - nqw;
    const int nb = int(sl.isQ ? a.nQblocks : a.nblocks - a.nQblocks);
    int bid = rel >> lg;
    sl.sub = rel & ((1 << lg) - 1);
    sl.valid = u < n_units && bid < nb;
    if (KIND == 1) bid = nb - 1 - bid;
    const int T_ = sl.isQ ? a.Tm : a.Tn;
    const int BLK_ = sl.isQ ? kPoolBQ : kPoolBK;
    const int bhi = sl.isQ ? fast_div(bid, a.tm_mul, a.tm_shr) : fast_div(bid, a.tn_mul, a.tn_shr);
    sl.bh = bhi;
    sl.blk = bid - bhi * T_;
    sl.rows = min(BLK_, a.N - sl.blk * BLK_);
    sl.srows = sl.valid ? max(0, min(SLAB, sl.rows - sl.sub * SLAB)) : 0;
    sl.row0 = sl.bh * a.N + int64_t(sl.blk) * BLK_ + sl.sub * SLAB;
    return sl;
  };
  // rows past the slab's end are filled with zeros (their source address is
  // the slab's block's first row, which every valid slab has, and is not read)
  auto prefetch = [&](const Slab& sl) {
    if (!PERSIST) return;
    if (sl.valid) {
      const uint16_t* base = static_cast<const uint16_t*>(sl.isQ ? a.q : a.k);
      const uint16_t* src = base + sl.row0 * D + c * 8;
      const uint16_t* blk0 = base + (sl.row0 - sl.sub * SLAB) * D + c * 8;
#pragma unroll
      for (int u = 0; u < NR; ++u) {
        const int r = ro + u * RPW;
        const bool in = r < sl.srows;
        cp_async16_zfill(&stage[warp][u][lane], in ? src + int64_t(r) * D : blk0, in ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  int64_t unit = blockIdx.x;
  Slab cur = slab_of(unit);
  prefetch(cur);
  for (; unit < n_units; unit += gridDim.x) {
  cp_async_wait_all();
  if (!cur.valid) {  // past the end: only the next unit's copies
    if (!PERSIST) break;
    cur = slab_of(unit + gridDim.x);
    prefetch(cur);
    continue;
  }
  const bool isQ = cur.isQ;
  const int G = isQ ? GQ : GK;
  const int sub = cur.sub;
  const int T = isQ ? a.Tm : a.Tn;
  const int64_t bh = cur.bh;
  const int blk = cur.blk;
  const int rows = cur.rows;
  const int srows = cur.srows;
  const int64_t row0 = cur.row0;

  uint4 raw[NR];
  if constexpr (PERSIST) {
#pragma unroll
    for (int u = 0; u < NR; ++u) raw[u] = stage[warp][u][lane];
  } else {
    const uint16_t* src = static_cast<const uint16_t*>(isQ ? a.q : a.k) + row0 * D + c * 8;
#pragma unroll
    for (int u = 0; u < NR; ++u) {
      const int r = ro + u * RPW;
      raw[u] = r < srows ? ld_stream(src + int64_t(r) * D) : make_uint4(0, 0, 0, 0);
    }
  }
  uint64_t nkb2[4];  // -kbar of this lane's 8 columns, as pairs
  if (KIND == 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      nkb2[e] = pack2(-a.kbar[bh * D + c * 8 + 2 * e], -a.kbar[bh * D + c * 8 + 2 * e + 1]);
  }

  float sx[8], su[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sx[e] = su[e] = 0.f;
  double s64[SUM64 ? 8 : 1];  // float64 column sums (KIND 2)
#pragma unroll
  for (int e = 0; e < (SUM64 ? 8 : 1); ++e) s64[e] = 0.0;
  float amax = 0.f;
  float inv_own[R];
  const int group_base = lane & ~(CH - 1);
  const int w0 = warp - sub;
  if (POOL) {
    // ---- pass 1: squared row norms (one value per row), column sums of x,
    // and the exact |x| max on the raw 16-bit halves
    float v[NR];
    uint64_t sx2[4];
    uint32_t am2[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) sx2[e] = pack2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < NR; ++u) {
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      uint64_t acc = pack2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint64_t x2 = widen2<BF16>(w[e]);
        acc = fma2(x2, x2, acc);
        sx2[e] = add2(sx2[e], x2);
        am2[e] = absmax2<BF16>(am2[e], w[e]);
      }
      float s0, s1;
      unpack2(acc, s0, s1);
      v[u] = s0 + s1;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) unpack2(sx2[e], sx[2 * e], sx[2 * e + 1]);
    amax = absmax2_value<BF16>(absmax2<BF16>(absmax2<BF16>(am2[0], am2[1]),
                                             absmax2<BF16>(am2[2], am2[3])));
    // ---- butterfly over the CH lanes of a row: at offset o the lanes with
    // bit o set keep the upper half of their rows and send the lower half;
    // once a lane is down to one row, the remaining offsets add plainly
#pragma unroll
    for (int o = CH / 2; o > 0; o >>= 1) {
      const bool up = (lane & o) != 0;
      const int cnt = NR * 2 * o / CH;  // rows carried into this step (< 2: one)
      if (cnt >= 2) {
#pragma unroll
        for (int k = 0; k < cnt / 2; ++k) {
          const float send = up ? v[k] : v[k + cnt / 2];
          const float keep = up ? v[k + cnt / 2] : v[k];
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
      }
    }
    // lane c of a row group now holds rows (c / SPREAD) * R .. + R - 1
#pragma unroll
    for (int t = 0; t < R; ++t) inv_own[t] = v[t] > 0.f ? rsqrtf(v[t]) : 0.f;
    if (SUM64) {
      // float64 column sums in a sweep of their own, once the row norms no
      // longer hold registers; rows past the block are zero and add nothing
#pragma unroll
      for (int u = 0; u < NR; ++u) {
        const uint4 rw = opaque(raw[u]);
        const uint32_t w[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x0, x1;
          unpack2(widen2<BF16>(w[e]), x0, x1);
          s64[2 * e] += f64_scaled(x0);
          s64[2 * e + 1] += f64_scaled(x1);
        }
      }
    }
  } else {
    // max |fl(x - kbar)| over the rows from each column's max and min of x:
    // rounding is monotone, so fl(xmin - kbar) <= fl(x - kbar) <= fl(xmax -
    // kbar) for every row, and the larger magnitude of those two is the max
    // (a lane's rows are valid in order: row u is valid only if row 0 is)
    uint32_t hi2[4], lo2[4];
#pragma unroll
    for (int u = 0; u < NR; ++u) {
      if (ro + u * RPW < srows) {
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi2[e] = u == 0 ? w[e] : max2_16<BF16>(hi2[e], w[e]);
          lo2[e] = u == 0 ? w[e] : min2_16<BF16>(lo2[e], w[e]);
        }
      }
    }
    if (ro < srows) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a0, a1, b0, b1;
        unpack2(add2(widen2<BF16>(hi2[e]), nkb2[e]), a0, a1);
        unpack2(add2(widen2<BF16>(lo2[e]), nkb2[e]), b0, b1);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a0), fabsf(a1)), fmaxf(fabsf(b0), fabsf(b1))));
      }
    }
  }
  // every loaded register has been read: the buffer takes the next unit
  if (PERSIST) prefetch(slab_of(unit + gridDim.x));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (POOL) {
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) sx[e] += __shfl_xor_sync(0xffffffffu, sx[e], o);
  }
  if (SUM64) {
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) s64[e] += __shfl_xor_sync(0xffffffffu, s64[e], o);
  }
  // ---- the block's absmax and column sums over its G slabs (slab order)
  if (G > 1) {
    if (POOL && ro == 0) {
      part8(warp, 0)[0] = make_float4(sx[0], sx[1], sx[2], sx[3]);
      part8(warp, 0)[1] = make_float4(sx[4], sx[5], sx[6], sx[7]);
    }
    if (SUM64 && ro == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) part64_8(warp)[e] = make_double2(s64[2 * e], s64[2 * e + 1]);
    }
    if (lane == 0) pmax[warp] = amax;
    named_barrier(1 + warp / G, 32 * G);
    if (POOL) {
      float4 lo = part8(w0, 0)[0], hi = part8(w0, 0)[1];
      for (int g = 1; g < G; ++g) {
        const float4 l2 = part8(w0 + g, 0)[0], h2 = part8(w0 + g, 0)[1];
        lo = make_float4(lo.x + l2.x, lo.y + l2.y, lo.z + l2.z, lo.w + l2.w);
        hi = make_float4(hi.x + h2.x, hi.y + h2.y, hi.z + h2.z, hi.w + h2.w);
      }
      sx[0] = lo.x, sx[1] = lo.y, sx[2] = lo.z, sx[3] = lo.w;
      sx[4] = hi.x, sx[5] = hi.y, sx[6] = hi.z, sx[7] = hi.w;
    }
    if (SUM64 && sub == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        double2 t = part64_8(w0)[e];
        for (int g = 1; g < G; ++g) {
          const double2 t2 = part64_8(w0 + g)[e];
          t.x += t2.x;
          t.y += t2.y;
        }
        s64[2 * e] = t.x;
        s64[2 * e + 1] = t.y;
      }
    }
    amax = pmax[w0];
    for (int g = 1; g < G; ++g) amax = fmaxf(amax, pmax[w0 + g]);
  }
  if (SUM64 && sub == 0 && ro == 0) {
    double* dst = a.ksum64 + (bh * T + blk) * D + c * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = s64[e] * kF64Unscale;
  }
  const bool quantise = KIND == 1 || (isQ && a.q_codes != nullptr);
  // delta = absmax / 127 (IEEE divide); inv = 1 / delta correctly rounded.  A
  // subnormal delta, whose reciprocal overflows, sends every code to the
  // exact path.
  const float delta = amax / 127.0f;
  const float inv = delta > 0.f ? __frcp_rn(delta) : 0.f;
  const bool exact_only = delta > 0.f && !(inv <= FLT_MAX);
  if (quantise && sub == 0 && lane == 0) (KIND == 1 ? a.dk : a.dq)[bh * T + blk] = delta;
  int8_t* codes = quantise ? (KIND == 1 ? a.k_codes : a.q_codes) + row0 * D + c * 8 : nullptr;
  // ---- pass 2: column sums of x / |x_row| (and the codes, once absmax is known)
  uint64_t su2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) su2[e] = pack2(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < NR; ++u) {
    const int r = ro + u * RPW;
    const uint4 rw = opaque(raw[u]);
    const uint32_t w[4] = {rw.x, rw.y, rw.z, rw.w};
    uint64_t x2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x2[e] = widen2<BF16>(w[e]);
    if (POOL) {
      const float iv = __shfl_sync(0xffffffffu, inv_own[u % R], group_base | ((u / R) * SPREAD));
      const uint64_t iv2 = pack2(iv, iv);
#pragma unroll
      for (int e = 0; e < 4; ++e) su2[e] = fma2(x2[e], iv2, su2[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) x2[e] = add2(x2[e], nkb2[e]);
    }
    if (quantise && r < srows)
      *reinterpret_cast<uint2*>(codes + int64_t(r) * D) = codes8(x2, inv, delta, exact_only);
  }
  if constexpr (POOL) {
#pragma unroll
    for (int e = 0; e < 4; ++e) unpack2(su2[e], su[2 * e], su[2 * e + 1]);
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) su[e] += __shfl_xor_sync(0xffffffffu, su[e], o);
    if (G > 1) {
      if (ro == 0) {
        part8(warp, D)[0] = make_float4(su[0], su[1], su[2], su[3]);
        part8(warp, D)[1] = make_float4(su[4], su[5], su[6], su[7]);
      }
      named_barrier(1 + warp / G, 32 * G);
      float4 lo = part8(w0, D)[0], hi = part8(w0, D)[1];
      for (int g = 1; g < G; ++g) {
        const float4 l2 = part8(w0 + g, D)[0], h2 = part8(w0 + g, D)[1];
        lo = make_float4(lo.x + l2.x, lo.y + l2.y, lo.z + l2.z, lo.w + l2.w);
        hi = make_float4(hi.x + h2.x, hi.y + h2.y, hi.z + h2.z, hi.w + h2.w);
      }
      su[0] = lo.x, su[1] = lo.y, su[2] = lo.z, su[3] = lo.w;
      su[4] = hi.x, su[5] = hi.y, su[6] = hi.z, su[7] = hi.w;
    }
    if (sub == 0) {
      float uu = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) uu = fmaf(su[e], su[e], uu);
#pragma unroll
      for (int o = CH / 2; o > 0; o >>= 1) uu += __shfl_xor_sync(0xffffffffu, uu, o);
      float* mean = isQ ? a.q_mean : a.k_mean;
      if (lane < CH) {
        // 1 / n is exact for a full block (a power of two), so this is sx / n
        const float rn = 1.0f / float(rows);
        float4* dst = reinterpret_cast<float4*>(mean + (bh * T + blk) * D + c * 8);
        dst[0] = make_float4(sx[0] * rn, sx[1] * rn, sx[2] * rn, sx[3] * rn);
        dst[1] = make_float4(sx[4] * rn, sx[5] * rn, sx[6] * rn, sx[7] * rn);
      }
      if (lane == 0) (isQ ? a.s_q : a.s_k)[bh * T + blk] = uu / (float(rows) * float(rows));
    }
  }
  if (!PERSIST) break;
  cur = slab_of(unit + gridDim.x);
  }
}

// kbar[bh, :] = fl32((sum over the N tokens of K[bh, :, :]) / N) with the sum
// in float64, in a fixed order.  One CTA per head and four adjacent columns
// (one 32-byte sector of a row of block sums): thread t takes column t % 4
// and the key blocks t / 4, t / 4 + 64, ...; the 64 partial sums of a column
// are then added by a butterfly within each warp and across the warps in
// warp order.  For 16-bit K every partial sum is exact (the exponents of
// realistic data span far fewer than 53 bits), so the result is the float64
// mean rounded once to float32, whatever the order.
constexpr int kKbarCols = 4;
__global__ void __launch_bounds__(256) kbar_kernel(const double* ksum, float* kbar, int32_t N,
                                                   int32_t Tn, int32_t D) {
  __shared__ double wsum[8][kKbarCols];
  const int groups = D / kKbarCols;
  const int64_t bh = blockIdx.x / groups;
  const int col = (blockIdx.x % groups) * kKbarCols + (threadIdx.x % kKbarCols);
  const int jl = threadIdx.x / kKbarCols, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double* src = ksum + bh * Tn * D + col;
  double acc = 0.0;
#pragma unroll 4
  for (int j = jl; j < Tn; j += 256 / kKbarCols) acc += src[int64_t(j) * D];
#pragma unroll
  for (int o = kKbarCols; o < 32; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane < kKbarCols) wsum[warp][lane] = acc;
  __syncthreads();
  if (threadIdx.x < kKbarCols) {
    double s = wsum[0][threadIdx.x];
#pragma unroll
    for (int w = 1; w < 8; ++w) s += wsum[w][threadIdx.x];
    kbar[bh * D + col] = __double2float_rn(s / double(N));
  }
}

// ------------------------------------------------------------------ select
constexpr int kSelRows = 8;                 // query blocks per CTA (one warp each)
constexpr int kSelThreads = kSelRows * 32;
constexpr int kSelCols = kSelThreads;       // key blocks scored per pass (one thread each)
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

// e * 2^38 as an integer (e in [0, 1]); exact for e >= 2^-14
__device__ __forceinline__ unsigned long long fixed38(float e) {
  return __float2ull_rz(e * 274877906944.0f);
}

__device__ __forceinline__ int visible_cols(int i, int N, int bq, int bk, int Tn, int causal) {
  if (!causal) return Tn;
  const int last_row = min(N, (i + 1) * bq) - 1;
  return min(Tn, last_row / bk + 1);
}

// A fix row (Eq. 9): every visible block of query block i is kept, in order.
// One warp.
__device__ __forceinline__ void write_full_row(const SelectArgs& a, int64_t bh, int i) {
  const int lane = threadIdx.x & 31;
  const int nvis = visible_cols(i, a.N, a.bq, a.bk, a.Tn, a.causal);
  const int64_t out = (bh * a.Tm + i) * a.Tn;
  for (int j = lane; j < a.Tn; j += 32) {
    a.mask[out + j] = j < nvis ? 1 : 0;
    if (j < nvis) a.kv_idx[out + j] = j;
  }
  if (lane == 0) a.kv_cnt[bh * a.Tm + i] = nvis;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
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

  // Eq. 9: a query block with s_q < theta is a fix block, its whole visible
  // row is 1 and its S_hat, softmax and TopCdf decide nothing.  When every
  // query block of this CTA is one, the S_hat phase is skipped.
  const bool my_fix = tid >= kSelRows || i0 + tid >= a.Tm ||
                      a.s_q[bh * a.Tm + i0 + tid] < a.theta;
  if (__syncthreads_and(my_fix)) {
    const int i = i0 + w;
    if (i < a.Tm) write_full_row(a, bh, i);
    return;
  }

  for (int idx = tid; idx < kSelRows * D; idx += kSelThreads) {
    const int r = idx / D, e = idx % D;
    qs[idx] = (i0 + r < a.Tm) ? a.q_mean[(bh * a.Tm + i0 + r) * D + e] : 0.f;
  }
  // ---- S_hat rows i0..i0+7 against every visible key block (Eq. 7, before
  // masking).  The key means stream through shared memory in chunks of
  // kSelCols blocks x 32 columns; each thread prefetches its share of the
  // next chunk into registers while the current one is multiplied, so the
  // L2 latency of the loads overlaps the arithmetic.
  const int njt = (jcount + kSelCols - 1) / kSelCols;
  const int nchunks = njt * (D / 32);
  float4 pre[kSelCols * 8 / kSelThreads];
  auto fetch = [&](int chunk) {
    const int jt = chunk / (D / 32), ec = (chunk % (D / 32)) * 32;
#pragma unroll
    for (int u = 0; u < kSelCols * 8 / kSelThreads; ++u) {
      const int idx = tid + u * kSelThreads;
      const int jl = idx >> 3, f4 = idx & 7, j = jt * kSelCols + jl;
      pre[u] = j < jcount
                   ? *reinterpret_cast<const float4*>(a.k_mean + (kbh * a.Tn + j) * D + ec + f4 * 4)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  if (nchunks > 0) fetch(0);
  float acc[kSelRows];
#pragma unroll
  for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
  for (int chunk = 0; chunk < nchunks; ++chunk) {
    const int jt = chunk / (D / 32), ec = (chunk % (D / 32)) * 32;
    __syncthreads();  // the previous chunk is no longer read
#pragma unroll
    for (int u = 0; u < kSelCols * 8 / kSelThreads; ++u) {
      const int idx = tid + u * kSelThreads;
      *reinterpret_cast<float4*>(ks + (idx >> 3) * kKPad + (idx & 7) * 4) = pre[u];
    }
    __syncthreads();
    if (chunk + 1 < nchunks) fetch(chunk + 1);
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
    if (ec + 32 == D) {
      const int j = jt * kSelCols + tid;
      if (j < jcount) {
#pragma unroll
        for (int r = 0; r < kSelRows; ++r) shat[r * a.Tn + j] = acc[r] * a.scale;
      }
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
    }
  }
  __syncthreads();

  // ---- one warp per query block: softmax, TopCdf, fix rule, compaction
  const int i = i0 + w;
  if (i >= a.Tm) return;
  float* row = shat + w * a.Tn;
  const int nvis = visible_cols(i, a.N, a.bq, a.bk, a.Tn, a.causal);
  const bool fix_row = a.s_q[bh * a.Tm + i] < a.theta;
  if (fix_row) {
    write_full_row(a, bh, i);
    return;
  }
  const float* sk = a.s_k + kbh * a.Tn;

  float mx = -INFINITY;
  for (int j = lane; j < nvis; j += 32) {
    const float v = sk[j] >= a.theta ? row[j] : -INFINITY;
    row[j] = v;
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  // unnormalised softmax weights; -1 marks a -inf entry.  Each weight's mass
  // is also taken as the integer e * 2^38 (exact for e >= 2^-14, below that
  // truncated by < 2^-38), so that every partial sum below is exact and does
  // not depend on the order of summation.
  unsigned long long tot = 0ull;
  for (int j = lane; j < nvis; j += 32) {
    const float v = row[j];
    const float e = (v == -INFINITY) ? -1.f : expf(v - mx);
    row[j] = e;
    if (e >= 0.f) tot += fixed38(e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  __syncwarp();
  float t_star = 0.f;  // keep e >= t_star (t_star = 0 keeps every finite entry)
  if (a.tau < 1.0f) {
    // t* = the largest row value t with sum_{e >= t} e >= tau * total, by a
    // radix select on the bit patterns of e (ordered like the values for
    // e >= 0), most significant byte first: each pass histograms the masses
    // of the entries that share the prefix found so far and picks the digit
    // where the running sum from the top reaches the target.
    const unsigned long long target =
        static_cast<unsigned long long>(ceil(double(a.tau) * double(tot)));
    // the warp's 256-bucket histogram of masses, as two 32-bit halves (the low
    // 19 bits of each mass and the rest, at most 2^19: a bucket's sums stay
    // below 5952 * 2^19 < 2^32 for the longest rows the library accepts), so
    // that every update is a native 32-bit shared atomic, not a 64-bit one
    uint32_t* hist_lo = reinterpret_cast<uint32_t*>(ks) + w * 512;
    uint32_t* hist_hi = hist_lo + 256;
    uint32_t prefix = 0u;
    unsigned long long above = 0ull;  // mass of the entries above the prefix's range
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      const uint32_t pmask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
#pragma unroll
      for (int b = 0; b < 8; ++b) hist_lo[lane * 8 + b] = hist_hi[lane * 8 + b] = 0u;
      __syncwarp();
      for (int j = lane; j < nvis; j += 32) {
        const float e = row[j];
        const uint32_t key = __float_as_uint(e);
        if (e >= 0.f && (key & pmask) == prefix) {
          const unsigned long long m = fixed38(e);
          const uint32_t bin = (key >> shift) & 255u;
          atomicAdd(hist_lo + bin, uint32_t(m & 0x7FFFFull));
          atomicAdd(hist_hi + bin, uint32_t(m >> 19));
        }
      }
      __syncwarp();
      // lane L holds digits 8L .. 8L+7; suffix sums over lanes from the top
      unsigned long long h[8], mine = 0ull;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        h[b] = (static_cast<unsigned long long>(hist_hi[lane * 8 + b]) << 19) + hist_lo[lane * 8 + b];
        mine += h[b];
      }
      unsigned long long incl = mine;  // mass of lanes >= this lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long up = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += up;
      }
      const unsigned ok = __ballot_sync(0xffffffffu, above + incl >= target);
      const int L = ok ? 31 - __clz(ok) : 0;  // the highest lane that reaches it
      uint32_t digit = 0u;
      unsigned long long run = above + incl - mine;  // mass above lane L's digits
      if (lane == L) {
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          if (run + h[b] >= target) {
            digit = uint32_t(8 * L + b);
            break;
          }
          run += h[b];
        }
      }
      digit = __shfl_sync(0xffffffffu, digit, L);
      above = __shfl_sync(0xffffffffu, run, L);
      prefix |= digit << shift;
      __syncwarp();
    }
    t_star = tot == 0ull ? INFINITY : __uint_as_float(prefix);
  }
  const int64_t out = (bh * a.Tm + i) * a.Tn;
  int cnt = 0;
  for (int jb = 0; jb < a.Tn; jb += 32) {
    const int j = jb + lane;
    bool keep = false;
    if (j < nvis) {
      const float e = row[j];
      keep = (e >= 0.f && e >= t_star) || sk[j] < a.theta;
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

// Persistent pooling grid: four CTAs per SM (the kernel's occupancy), no more
// than there are units of work (one CTA per unit for the K pooling pass).  The
// shared-memory carveout is set to its maximum so that four CTAs' slab
// buffers fit.
template <int D, bool BF16, int KIND, int SLAB>
cudaError_t launch_pool(const PoolArgs& pa, int64_t warps, cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pool_kernel<D, BF16, KIND, SLAB>,
                           cudaFuncAttributePreferredSharedMemoryCarveout,
                           int(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  constexpr int WARPS = pool_warps(SLAB);
  const int64_t units = cdiv(warps, WARPS);
  const int64_t ctas = KIND == 2 ? units
                                 : std::max<int64_t>(1, std::min<int64_t>(
                                                            units, int64_t(sms) * pool_min_blocks(SLAB)));
  pool_kernel<D, BF16, KIND, SLAB><<<unsigned(ctas), 32 * WARPS, 0, s>>>(pa);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t pool_impl(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  if (p.bq != kPoolBQ || p.bk != kPoolBK) return cudaErrorInvalidValue;
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
  PoolArgs pa{};
  pa.q = x.q;
  pa.k = x.k;
  pa.N = p.N;
  pa.bq = p.bq;
  pa.bk = p.bk;
  pa.Tm = int32_t(Tm);
  pa.Tn = int32_t(Tn);
  const FastDiv dm = FastDiv::make(uint32_t(Tm)), dn = FastDiv::make(uint32_t(Tn));
  pa.tm_mul = dm.mul;
  pa.tm_shr = dm.shr;
  pa.tn_mul = dn.mul;
  pa.tn_shr = dn.shr;
  const int64_t nK = int64_t(p.B) * p.Hkv * Tn;
  pa.nQblocks = int64_t(p.B) * p.Hq * Tm;
  pa.nblocks = pa.nQblocks + nK;
  pa.q_mean = x.q_mean;
  pa.k_mean = x.k_mean;
  pa.s_q = x.s_q;
  pa.s_k = x.s_k;
  pa.q_codes = x.q_codes;
  pa.dq = x.dq;
  pa.status = x.status;
  cudaError_t e;
  constexpr int SLAB = D == 128 ? 32 : 64;  // 8 KB of bf16/f16 per warp
  constexpr int SLAB_Q = SLAB;  // the pooling pass's slab (any power of two from 16 works)
  constexpr int64_t GK = kPoolBK / SLAB;
  constexpr int64_t GQq = kPoolBQ / SLAB_Q, GKq = kPoolBK / SLAB_Q;
  if (x.k_codes == nullptr) {
    // one pass over Q then K blocks
    return launch_pool<D, BF16, 0, SLAB_Q>(pa, pa.nQblocks * GQq + nK * GKq, s);
  }
  if constexpr (D != 128) {
    return cudaErrorInvalidValue;  // the INT8 path exists for d = 128 only
  } else {
  // INT8: K first -- pooling with float64 column sums, kbar, then the codes of
  // K - kbar (last blocks first, while they are still in L2) -- then Q's
  // pooling pass, which also writes the Q codes.
  PoolArgs ka = pa;
  ka.nQblocks = 0;
  ka.nblocks = nK;
  ka.ksum64 = x.ksum64;
  if ((e = launch_pool<D, BF16, 2, SLAB>(ka, nK * GK, s)) != cudaSuccess) return e;
  kbar_kernel<<<unsigned(int64_t(p.B) * p.Hkv * (D / kKbarCols)), 256, 0, s>>>(
      x.ksum64, x.kbar, p.N, int32_t(Tn), D);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  PoolArgs ca = ka;
  ca.kbar = x.kbar;
  ca.k_codes = x.k_codes;
  ca.dk = x.dk;
  if ((e = launch_pool<D, BF16, 1, SLAB>(ca, nK * GK, s)) != cudaSuccess) return e;
  PoolArgs qa = pa;
  qa.nblocks = qa.nQblocks;
  return launch_pool<D, BF16, 0, SLAB_Q>(qa, qa.nQblocks * GQq, s);
  }
}

template <int D>
cudaError_t select_impl(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
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
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem));
  if (e != cudaSuccess) return e;
  dim3 sgrid{unsigned(cdiv(Tm, kSelRows)), unsigned(p.Hq), unsigned(p.B)};
  select_kernel<D><<<sgrid, kSelThreads, smem, s>>>(sa);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_predict_pool(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  const bool bf16 = p.io_dtype == SPARGE_BF16;
  if (p.d == 128) return bf16 ? pool_impl<128, true>(p, x, s) : pool_impl<128, false>(p, x, s);
  if (p.d == 64) return bf16 ? pool_impl<64, true>(p, x, s) : pool_impl<64, false>(p, x, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_predict_select(const sparge_params_t& p, const PredictPtrs& x,
                                  cudaStream_t s) {
  if (p.d == 128) return select_impl<128>(p, x, s);
  if (p.d == 64) return select_impl<64>(p, x, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_predict(const sparge_params_t& p, const PredictPtrs& x, cudaStream_t s) {
  const cudaError_t e = launch_predict_pool(p, x, s);
  return e != cudaSuccess ? e : launch_predict_select(p, x, s);
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
