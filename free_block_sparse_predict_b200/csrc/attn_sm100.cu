// Stage 2 of SpargeAttn on sm_100a: block-sparse online-softmax attention
// (paper review page, section 三: Eq. 1 online softmax, Eq. 2 block skip,
// Eq. 3 and "Sparse Warp Online Softmax" per-warp P~V skip; Algorithm 1
// steps 6-17), with the optional per-block INT8 Q K^T of steps 2 and 10.
//
// One CTA per 128-row query tile (b, h, i), 192 threads:
//   warp 0     TMA producer: Q tile once, then K_j / V_j of the tile's skip
//              list into rings of shared-memory stages (128B swizzle), K
//              running ahead of V.
//   warp 1     allocates tensor memory; one thread issues every tcgen05.mma:
//              S_t = Q K_t^T into a double-buffered S (TMEM), and
//              O += P~_t V_t with P~ read from TMEM (aliased over S_t).
//   warps 2-5  softmax: thread r owns query row r (its TMEM lane).  Per key
//              block: masks, running max, the lambda vote of its warp's 32
//              rows (Eq. 3), P~ in fp16 back into TMEM, the row sum l, and a
//              lazy rescale of its O row when the max grows by > 2^8.  The
//              epilogue divides by l and stores O.
// Pairs of CTAs share an SM (<= 113 KB shared memory, 256 TMEM columns each),
// so one CTA's softmax overlaps the other's tensor-core work.
//
// Every mbarrier wait is bounded; a timeout sets the workspace status word to
// SPARGE_ETIMEOUT, stops all roles, lets outstanding copies land, frees the
// tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "sm100_ptx.cuh"
#include "sparge_internal.h"

namespace sparge {
namespace {

constexpr int kBQ = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

enum QKMode { kF16 = 0, kBF16 = 1, kI8 = 2 };

template <int D, int MODE>
struct Cfg {
  static constexpr int QK_ES = MODE == kI8 ? 1 : 2;           // bytes per Q/K element
  static constexpr int BOX_X = 128 / QK_ES;                   // elements per 128-byte row
  static constexpr int QK_BOXES = D / BOX_X;                  // 128-byte column slabs of Q/K
  static constexpr int V_BOXES = D / 64;                      // 128-byte column slabs of V
  static constexpr int Q_BYTES = kBQ * D * QK_ES;
  static constexpr int K_BYTES = kBK * D * QK_ES;
  static constexpr int V_BYTES = kBK * D * 2;
  // K_t is needed by S_t one block before V_t is needed by P~_t V_t, so K may
  // run further ahead where shared memory allows (16-bit d = 128: 2 + 2
  // stages; a third K stage there measured no faster).
  static constexpr int K_STAGES = (D == 64) ? 6 : (MODE == kI8 ? 4 : 2);
  static constexpr int V_STAGES = (D == 64) ? 4 : (MODE == kI8 ? 3 : 2);
  static constexpr int KSTEP = MODE == kI8 ? 32 : 16;         // MMA K per instruction
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int TMEM_COLS = 256;                       // S0 | S1 | O
  static constexpr int O_COL = 128;
  static constexpr int SMEM_TILES = Q_BYTES + K_STAGES * K_BYTES + V_STAGES * V_BYTES;
  static constexpr int SMEM_BYTES = SMEM_TILES + 256 /*barriers*/;
  // two CTAs per SM: 228 KB of shared memory, 1 KB of it reserved per CTA
  static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");
};

struct AttnParams {
  CUtensorMap tmQ;
  CUtensorMap tmK;
  CUtensorMap tmV;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  void* o;
  const float* dq;
  const float* dk;
  int32_t* status;
  sparge_stats_t* stats;
  int32_t B, Hq, Hkv, N, Tm, Tn, causal, o_f32, o_bf16;
  float scale_log2;  // scale * log2(e)
  float lam2;        // lambda * log2(e)
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[6], k_empty[6], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final;
  uint32_t skip[2];  // byte q = 1 when softmax warp of quadrant q skips P~V
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(Bars) <= 256, "barrier block");

__device__ __forceinline__ void report_timeout(int32_t* status, volatile int* abort) {
  *abort = 1;
  atomicExch(status, int32_t(SPARGE_ETIMEOUT));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max of 64 floats (given as bits) by a depth-4 tree of three-input maxima
__device__ __forceinline__ float max64(const uint32_t (&v)[64]) {
  float a[22], b[8];
#pragma unroll
  for (int c = 0; c < 21; ++c)
    a[c] = fmax3(__uint_as_float(v[3 * c]), __uint_as_float(v[3 * c + 1]),
                 __uint_as_float(v[3 * c + 2]));
  a[21] = __uint_as_float(v[63]);
#pragma unroll
  for (int c = 0; c < 7; ++c) b[c] = fmax3(a[3 * c], a[3 * c + 1], a[3 * c + 2]);
  b[7] = a[21];
  return fmax3(fmax3(b[0], b[1], b[2]), fmax3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 2) attn_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<D, MODE>;
  // 128-byte-swizzled tiles need 1024-byte alignment; the dynamic shared
  // memory of a kernel without static shared memory starts there.  Checked,
  // not assumed: a misplaced window reports SPARGE_EUNSUPPORTED.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(P.status, 0, int32_t(SPARGE_EUNSUPPORTED));
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;
  uint8_t* sV = sK + C::K_STAGES * C::K_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(sV + C::V_STAGES * C::V_BYTES);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- tile of this CTA.  Tiles are ordered by (batch, KV head) first, so
  // the CTAs resident at any time read the K/V of one KV head, which then
  // stays in L2 (50 MB at N = 128K, d = 128) instead of all heads' streaming
  // through it; within a KV head, heavy (late) query blocks first, and the
  // query heads of the group adjacent.
  const int G = P.Hq / P.Hkv;
  const int64_t per_kv = int64_t(P.Tm) * G;
  const int64_t bhk = blockIdx.x / per_kv;
  const int64_t rem = blockIdx.x % per_kv;
  const int i = P.Tm - 1 - int(rem / G);
  const int b = int(bhk / P.Hkv), hk = int(bhk % P.Hkv);
  const int h = hk * G + int(rem % G);
  const int64_t bh = int64_t(b) * P.Hq + h;
  const int64_t tile = bh * P.Tm + i;
  const int32_t* kv_list = P.kv_idx + tile * P.Tn;
  int n = P.kv_cnt[tile];
  n = n < 0 ? 0 : (n > P.Tn ? P.Tn : n);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::K_STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::V_STAGES; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 4);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_final, 1);
    bars->skip[0] = bars->skip[1] = 0;
    bars->abort = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // =================================================== TMA producer
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&P.tmQ);
      tma_prefetch_desc(&P.tmK);
      tma_prefetch_desc(&P.tmV);
      int k_issued[C::K_STAGES] = {}, v_issued[C::V_STAGES] = {};
      mbar_expect_tx(&bars->q_full, C::Q_BYTES);
      for (int x = 0; x < C::QK_BOXES; ++x)
        tma_load_3d(sQ + x * (kBQ * 128), &P.tmQ, &bars->q_full, x * C::BOX_X, i * kBQ,
                    int32_t(bh));
      // K_t into stage t % K_STAGES once Q K_{t-K_STAGES}^T has read it
      auto load_k = [&](int t) -> bool {
        const int st = t % C::K_STAGES, use = t / C::K_STAGES;
        if (use > 0 && !mbar_wait(&bars->k_empty[st], (use - 1) & 1, abort, P.status)) return false;
        const int j = __ldg(kv_list + t);
        mbar_expect_tx(&bars->k_full[st], C::K_BYTES);
        for (int x = 0; x < C::QK_BOXES; ++x)
          tma_load_3d(sK + st * C::K_BYTES + x * (kBK * 128), &P.tmK, &bars->k_full[st],
                      x * C::BOX_X, j * kBK, int32_t(bhk));
        ++k_issued[st];
        return true;
      };
      // V_t once P~_{t-V_STAGES} V_{t-V_STAGES} has read its stage
      auto load_v = [&](int t) -> bool {
        const int st = t % C::V_STAGES, use = t / C::V_STAGES;
        if (use > 0 && !mbar_wait(&bars->v_empty[st], (use - 1) & 1, abort, P.status)) return false;
        const int j = __ldg(kv_list + t);
        mbar_expect_tx(&bars->v_full[st], C::V_BYTES);
        for (int x = 0; x < C::V_BOXES; ++x)
          tma_load_3d(sV + st * C::V_BYTES + x * (kBK * 128), &P.tmV, &bars->v_full[st], x * 64,
                      j * kBK, int32_t(bhk));
        ++v_issued[st];
        return true;
      };
      // K runs K_STAGES blocks ahead of V: the tensor pipe needs K_{t+1} (for
      // S_{t+1}) before V_t (for P~_t V_t).  V_t waits for P~V of block
      // t - V_STAGES, which the tensor pipe runs before S_t, whose end frees
      // the stage of K_{t+K_STAGES}: so a V wait never holds K back.
      bool ok = true;
      for (int t = 0; t < n && t < C::K_STAGES && ok; ++t) ok = load_k(t);
      for (int t = 0; t < n && ok; ++t) {
        ok = load_v(t);
        if (ok && t + C::K_STAGES < n) ok = load_k(t + C::K_STAGES);
      }
      if (!ok) report_timeout(P.status, abort);
      // let every copy this thread started land before the CTA can exit
      mbar_wait_teardown(&bars->q_full, 0);
      for (int s = 0; s < C::K_STAGES; ++s)
        if (k_issued[s] > 0) mbar_wait_teardown(&bars->k_full[s], (k_issued[s] - 1) & 1);
      for (int s = 0; s < C::V_STAGES; ++s)
        if (v_issued[s] > 0) mbar_wait_teardown(&bars->v_full[s], (v_issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    // =================================================== MMA issuer
    if (lane == 0 && n > 0) {
      const uint32_t idesc_qk =
          MODE == kI8 ? instr_desc(2, 1, 1, 0, kBQ, kBK) : instr_desc(1, MODE, MODE, 0, kBQ, kBK);
      const uint32_t idesc_pv = instr_desc(1, 0, 0, 1, kBQ, D);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      uint32_t pv_count = 0;
      bool ok = mbar_wait(&bars->q_full, 0, abort, P.status);
      tc_fence_after();
      auto do_pv = [&](int u) -> bool {
        const int sb = u & 1;
        if (!mbar_wait(&bars->p_full[sb], (u >> 1) & 1, abort, P.status)) return false;
        tc_fence_after();
        const uint32_t flags = *reinterpret_cast<volatile uint32_t*>(&bars->skip[sb]);
        const int stv = u % C::V_STAGES;
        if (!mbar_wait(&bars->v_full[stv], (u / C::V_STAGES) & 1, abort, P.status)) return false;
        tc_fence_after();
        if (flags != 0x01010101u) {
          const uint32_t a_tmem = tmem + uint32_t(sb * kBK);
          const uint32_t vbase = sVa + uint32_t(stv * C::V_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc(vbase + kk * 2048, kBK * 128, 1024);
            mma_f16_ts(tmem + C::O_COL, a_tmem + kk * 8, bdesc, idesc_pv,
                       (pv_count > 0 || kk > 0) ? 1u : 0u);
          }
          ++pv_count;
        }
        mma_commit(&bars->v_empty[stv]);
        mma_commit(&bars->o_done);
        return true;
      };
      for (int t = 0; t < n && ok; ++t) {
        const int st = t % C::K_STAGES;
        if (!(ok = mbar_wait(&bars->k_full[st], (t / C::K_STAGES) & 1, abort, P.status))) break;
        tc_fence_after();
        const int sb = t & 1;
        const uint32_t kbase = sKa + uint32_t(st * C::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
          const int slab = (kk * C::KSTEP) / C::BOX_X;
          const int within = ((kk * C::KSTEP) % C::BOX_X) * C::QK_ES;
          const uint64_t adesc = smem_desc(sQa + slab * (kBQ * 128) + within, 16, 1024);
          const uint64_t bdesc = smem_desc(kbase + slab * (kBK * 128) + within, 16, 1024);
          if (MODE == kI8)
            mma_i8_ss(tmem + uint32_t(sb * kBK), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
          else
            mma_f16_ss(tmem + uint32_t(sb * kBK), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->k_empty[st]);
        if (t >= 1) ok = do_pv(t - 1);
      }
      if (ok) ok = do_pv(n - 1);
      if (!ok) report_timeout(P.status, abort);
      mma_commit(&bars->o_final);
      if (!ok) {
        // wait for the MMAs already issued before the memory is released
        mbar_wait_teardown(&bars->o_final, 0);
      }
      if (P.stats != nullptr) {
        atomicAdd(&P.stats->qk_blocks, (unsigned long long)n);
        atomicAdd(&P.stats->pv_blocks, (unsigned long long)pv_count);
      }
    }
    if (lane == 0 && P.stats != nullptr) atomicAdd(&P.stats->tiles, 1ull);
  } else {
    // =================================================== softmax warps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int row_g = i * kBQ + r;
    const bool row_ok = row_g < P.N;
    const bool slice_exists = i * kBQ + quad * 32 < P.N;
    const uint32_t lane_addr = tmem + (uint32_t(quad * 32) << 16);
    const float dq_i = MODE == kI8 ? P.dq[bh * P.Tm + i] : 1.f;
    float m_true = -INFINITY, m_sc = -INFINITY, l = 0.f;
    bool issued_any = false;
    uint32_t kept_slices = 0, skipped_slices = 0;
    bool ok = true;
    // skip-list index (and INT8 block scale) one block ahead of their use
    int j_next = n > 0 ? __ldg(kv_list) : 0;
    for (int t = 0; t < n; ++t) {
      const int sb = t & 1;
      const int j = j_next;
      float sc = P.scale_log2;
      if (MODE == kI8)
        sc *= dq_i * (uint32_t(j) < uint32_t(P.Tn) ? __ldg(P.dk + bhk * P.Tn + j) : 0.f);
      if (t + 1 < n) j_next = __ldg(kv_list + t + 1);
      // keys c < lim of this block exist for this row (past N, causal future
      // and rows past N are masked)
      const int key0 = j * kBK;
      int lim = P.N - key0;
      if (P.causal) lim = min(lim, row_g - key0 + 1);
      if (!row_ok || j < 0) lim = 0;

      // the outcome of every wait is made warp-uniform before it steers control
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (t >> 1) & 1, abort, P.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t raw[64];
      {
        uint32_t (&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&raw[0]);
        uint32_t (&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&raw[32]);
        tmem_ld32(lane_addr + uint32_t(sb * kBK), r0);
        tmem_ld32(lane_addr + uint32_t(sb * kBK + 32), r1);
        // the fenced waits tie r0 / r1 to the wait, so no use of them can be
        // scheduled before the loads have landed
        tmem_wait_ld_fence(r0);
        tmem_wait_ld_fence(r1);
      }
      // INT8 scores become floats first, without the conversion unit (it
      // shares the MUFU pipe with ex2): the bits of 1.5 * 2^23 + x are that
      // float exactly for |x| < 2^22, and an INT8 score of d = 128 is at most
      // 127^2 * 128; the order of x is kept, so the max runs on them as is.
      constexpr float kMagic = 12582912.0f;
      if (MODE == kI8) {
#pragma unroll
        for (int c = 0; c < 64; ++c) raw[c] += 0x4B400000u;
      }
      if (lim < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= lim) raw[c] = 0xFF800000u;  // -inf
      }
      // row max on the raw accumulators (sc > 0 preserves the order), by a
      // tree of three-input maxima
      const float m_raw = max64(raw);
      // (an INT8 block scale can be 0: keep an all-masked row at -inf)
      const float m_loc =
          m_raw == -INFINITY ? -INFINITY : (MODE == kI8 ? m_raw - kMagic : m_raw) * sc;
      const float m_new = fmaxf(m_true, m_loc);
      const float diff = (m_loc == -INFINITY) ? -INFINITY : (m_loc - m_new);
      const bool skip = __all_sync(0xffffffffu, diff < P.lam2);
      // lazy rescale of the O row once the max has grown by more than 2^8
      const bool grow = m_new > m_sc + kRescaleThreshold;
      const bool need_o = grow && (m_sc != -INFINITY);
      if (__any_sync(0xffffffffu, need_o)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (t - 1) & 1, abort, P.status));
        if (!ok) break;
        tc_fence_after();
        const float alpha = need_o ? ex2_approx(m_sc - m_new) : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_addr + uint32_t(C::O_COL + cc * 32), o);
          tmem_wait_ld_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_addr + uint32_t(C::O_COL + cc * 32), o);
        }
        if (need_o) l *= alpha;
      }
      if (grow) m_sc = m_new;
      // P~ = 2^(x * sc - m_sc): one packed FMA per pair, then ex2 on the MUFU
      const float nb = (m_sc == -INFINITY) ? 0.f : -m_sc;
      const uint64_t sc2 = pack2(sc, sc), nb2 = pack2(nb, nb);
      float pv[64];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        uint64_t x2 = pack2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
        if (MODE == kI8) x2 = add2(x2, pack2(-kMagic, -kMagic));  // exact
        float y0, y1;
        unpack2(fma2(x2, sc2, nb2), y0, y1);
        pv[c] = ex2_approx(y0);
        pv[c + 1] = ex2_approx(y1);
      }
      if (lim < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= lim) pv[c] = 0.f;
      }
      // row sum by a packed tree
      uint64_t acc[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        acc[c] = add2(pack2(pv[2 * c], pv[2 * c + 1]), pack2(pv[2 * c + 32], pv[2 * c + 33]));
#pragma unroll
      for (int w2 = 8; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int c = 0; c < w2; ++c) acc[c] = add2(acc[c], acc[c + w2]);
      float rs0, rs1;
      unpack2(acc[0], rs0, rs1);
      l += rs0 + rs1;
      m_true = m_new;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) pk[c] = skip ? 0u : pack_half2(pv[2 * c], pv[2 * c + 1]);
      tmem_st32(lane_addr + uint32_t(sb * kBK), pk);
      tmem_wait_st();
      if (!skip) issued_any = true;
      if (slice_exists) {
        if (skip) ++skipped_slices; else ++kept_slices;
      }
      if (lane == 0) reinterpret_cast<volatile uint8_t*>(&bars->skip[sb])[quad] = skip ? 1 : 0;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[sb]);
    }
    if (!ok) report_timeout(P.status, abort);
    // ---- epilogue: O / l
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0, abort, P.status));
    if (!ok) report_timeout(P.status, abort);
    tc_fence_after();
    if (ok) {
      const bool valid = issued_any && l > 0.f && n > 0;
      const float inv_l = valid ? 1.f / l : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32] = {};
        if (n > 0) {
          tmem_ld32(lane_addr + uint32_t(C::O_COL + cc * 32), o);
          tmem_wait_ld_fence(o);
        }
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = valid ? __uint_as_float(o[e]) * inv_l : 0.f;
        if (row_ok) {
          const int64_t off = (bh * P.N + row_g) * D + cc * 32;
          if (P.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.o) + off);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (P.o_bf16) {
                __nv_bfloat162 t2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                w[e] = *reinterpret_cast<uint32_t*>(&t2);
              } else {
                w[e] = pack_half2(v[2 * e], v[2 * e + 1]);
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.o) + off);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
      }
    }
    if (P.stats != nullptr) {
      if (lane == 0 && (kept_slices | skipped_slices)) {
        atomicAdd(&P.stats->pv_slices, (unsigned long long)kept_slices);
        atomicAdd(&P.stats->skipped_slices, (unsigned long long)skipped_slices);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// bf16 -> f16 copy of V for the fp16 P~V product; values beyond the fp16
// range are saturated and flagged with SPARGE_ERANGE.
__global__ void v_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                int64_t n16, int32_t* status) {
  bool bad = false;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < n16;
       t += int64_t(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(src + t);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
      if (fabsf(lo) > 65504.f || fabsf(hi) > 65504.f) bad = true;
      lo = fminf(65504.f, fmaxf(-65504.f, lo));
      hi = fminf(65504.f, fmaxf(-65504.f, hi));
      o[e] = pack_half2(lo, hi);
    }
    dst[t] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
    atomicCAS(status, 0, int32_t(SPARGE_ERANGE));
}

// --------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn query_encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// looked up once; the initialisation of a function-local static is
// thread-safe, so concurrent first calls from several host threads are fine
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = query_encode_fn();
  return fn;
}

// [BH, N, D] row-major tensor; box of box_x elements x rows x 1, 128B swizzle.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int es, const void* base, int D, int N,
              int64_t BH, int box_x, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * es, cuuint64_t(N) * D * es};
  cuuint32_t box[3] = {cuuint32_t(box_x), cuuint32_t(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int MODE>
cudaError_t attn_impl(const sparge_params_t& p, const AttnPtrs& x, cudaStream_t s) {
  using C = Cfg<D, MODE>;
  AttnParams P;
  memset(&P, 0, sizeof(P));
  const int64_t Tm = cdiv(p.N, p.bq), Tn = cdiv(p.N, p.bk);
  const CUtensorMapDataType qk_dt = MODE == kI8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : MODE == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_map(&P.tmQ, qk_dt, C::QK_ES, x.q, D, p.N, int64_t(p.B) * p.Hq, C::BOX_X, kBQ) ||
      !make_map(&P.tmK, qk_dt, C::QK_ES, x.k, D, p.N, int64_t(p.B) * p.Hkv, C::BOX_X, kBK) ||
      !make_map(&P.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x.v, D, p.N, int64_t(p.B) * p.Hkv,
                64, kBK))
    return cudaErrorNotSupported;
  P.kv_idx = x.kv_idx;
  P.kv_cnt = x.kv_cnt;
  P.o = x.o;
  P.dq = x.dq;
  P.dk = x.dk;
  P.status = x.status;
  P.stats = x.stats;
  P.B = p.B;
  P.Hq = p.Hq;
  P.Hkv = p.Hkv;
  P.N = p.N;
  P.Tm = int32_t(Tm);
  P.Tn = int32_t(Tn);
  P.causal = p.causal;
  P.o_f32 = p.o_dtype == SPARGE_F32;
  P.o_bf16 = p.o_dtype == SPARGE_BF16;
  P.scale_log2 = p.scale * kLog2e;
  P.lam2 = std::isinf(p.lambda) ? p.lambda : p.lambda * kLog2e;
  cudaError_t e;
  if (x.v16 != nullptr) {
    const int64_t n16 = int64_t(p.B) * p.Hkv * p.N * p.d / 8;
    int64_t blocks = cdiv(n16, 256 * 4);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    v_to_f16_kernel<<<unsigned(blocks), 256, 0, s>>>(static_cast<const uint4*>(x.v_io),
                                                     static_cast<uint4*>(x.v16), n16, x.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(attn_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t tiles = int64_t(p.B) * p.Hq * Tm;
  attn_kernel<D, MODE><<<unsigned(tiles), kThreads, C::SMEM_BYTES, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const sparge_params_t& p, const AttnPtrs& x, cudaStream_t s) {
  if (p.qk_int8) {
    if (p.d == 128) return attn_impl<128, kI8>(p, x, s);
    return cudaErrorInvalidValue;
  }
  const bool bf16 = p.io_dtype == SPARGE_BF16;
  if (p.d == 128) return bf16 ? attn_impl<128, kBF16>(p, x, s) : attn_impl<128, kF16>(p, x, s);
  if (p.d == 64) return bf16 ? attn_impl<64, kBF16>(p, x, s) : attn_impl<64, kF16>(p, x, s);
  return cudaErrorInvalidValue;
}

}  // namespace sparge
