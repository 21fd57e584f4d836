// Hilbert-curve token permutation (paper review page, section 三 "HilbertCurve
// Permutation"; rebuttal page, reply to Weakness 3): visual tokens of a
// T x H x W grid are reordered along a Hilbert curve so that spatial
// neighbours share query/key blocks, and the output is put back afterwards.
//
// The table is built on the device by walking the curve: every position h of
// the 2^(n*b) cube is decoded to grid coordinates with Skilling's transpose
// algorithm ("Programming the Hilbert curve", AIP Conf. Proc. 707, 2004, the
// index-to-axes direction), positions outside the grid are dropped, and an
// exclusive scan over the survivors gives each grid token its rank.  The
// gather / scatter kernels then move whole 16-byte chunks of token rows.
#include <cstdint>
#include <type_traits>

#include "sparge_internal.h"

namespace sparge {
namespace {

constexpr int kHilThreads = 256;
constexpr int kHilPerThread = 4;
constexpr int kHilPerCta = kHilThreads * kHilPerThread;

struct HilbertGrid {
  int32_t n;        // curve dimensions (axes of extent > 1)
  int32_t bits;     // cube side 2^bits
  int32_t ext[3];   // extents of the curve axes, in (t, y, x) order
  int32_t mul[3];   // linear-index multiplier of each curve axis
  int64_t cube;     // 2^(n*bits)
};

// Curve position -> grid coordinates (transpose form, Gray decode, undo), for
// a curve of NA axes: the axis loops unroll, so the coordinates stay in
// registers.  h < 2^(NA * bits) <= 2^30.
template <int NA>
__device__ __forceinline__ bool hilbert_decode(const HilbertGrid& g, uint32_t h, int32_t* lin) {
  uint32_t X[NA];
#pragma unroll
  for (int i = 0; i < NA; ++i) X[i] = 0;
  for (int l = 0; l < g.bits; ++l) {
#pragma unroll
    for (int i = 0; i < NA; ++i) X[i] |= ((h >> (l * NA + NA - 1 - i)) & 1u) << l;
  }
  uint32_t t = X[NA - 1] >> 1;
#pragma unroll
  for (int i = NA - 1; i > 0; --i) X[i] ^= X[i - 1];
  X[0] ^= t;
  for (uint32_t Q = 2; Q != (1u << g.bits); Q <<= 1) {
    const uint32_t P = Q - 1;
#pragma unroll
    for (int i = NA - 1; i >= 0; --i) {
      if (X[i] & Q) {
        X[0] ^= P;
      } else {
        t = (X[0] ^ X[i]) & P;
        X[0] ^= t;
        X[i] ^= t;
      }
    }
  }
  int32_t L = 0;
#pragma unroll
  for (int i = 0; i < NA; ++i) {
    if (X[i] >= uint32_t(g.ext[i])) return false;
    L += int32_t(X[i]) * g.mul[i];
  }
  *lin = L;
  return true;
}

template <int NA>
__global__ void hilbert_count_kernel(HilbertGrid g, int32_t* counts) {
  const int64_t base = int64_t(blockIdx.x) * kHilPerCta;
  int c = 0;
#pragma unroll
  for (int k = 0; k < kHilPerThread; ++k) {
    const int64_t h = base + int64_t(threadIdx.x) * kHilPerThread + k;
    int32_t lin;
    if (h < g.cube && hilbert_decode<NA>(g, uint32_t(h), &lin)) ++c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  __shared__ int sh[kHilThreads / 32];
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int i = 0; i < kHilThreads / 32; ++i) s += sh[i];
    counts[blockIdx.x] = s;
  }
}

template <int NA>
__global__ void hilbert_scatter_kernel(HilbertGrid g, const int32_t* counts, int32_t ncount,
                                       int32_t N, int32_t prefix_len, int32_t L, int32_t* perm) {
  __shared__ int sh[kHilThreads / 32];
  __shared__ int s_base;
  // offset of this CTA = survivors of all earlier CTAs
  int pre = 0;
  const int upto = min(int(blockIdx.x), ncount);
  for (int i = threadIdx.x; i < upto; i += kHilThreads) pre += counts[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, o);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = pre;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int i = 0; i < kHilThreads / 32; ++i) s += sh[i];
    s_base = s;
  }
  __syncthreads();
  // survivors of this thread, then an exclusive scan across the CTA
  const int64_t base = int64_t(blockIdx.x) * kHilPerCta + int64_t(threadIdx.x) * kHilPerThread;
  int32_t lin[kHilPerThread];
  bool in[kHilPerThread];
  int c = 0;
#pragma unroll
  for (int k = 0; k < kHilPerThread; ++k) {
    const int64_t h = base + k;
    in[k] = h < g.cube && hilbert_decode<NA>(g, uint32_t(h), &lin[k]);
    c += in[k];
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  __syncthreads();
  if (lane == 31) sh[w] = incl;
  __syncthreads();
  int warp_off = 0;
  for (int i = 0; i < w; ++i) warp_off += sh[i];
  int rank = s_base + warp_off + incl - c;
#pragma unroll
  for (int k = 0; k < kHilPerThread; ++k) {
    if (in[k]) {
      if (rank < L) perm[prefix_len + rank] = prefix_len + lin[k];
      ++rank;
    }
  }
  // tokens outside the grid keep their place
  const int64_t stride = int64_t(gridDim.x) * kHilThreads;
  for (int64_t p = int64_t(blockIdx.x) * kHilThreads + threadIdx.x; p < N; p += stride)
    if (p < prefix_len || p >= prefix_len + L) perm[p] = int32_t(p);
}

// Whole-row gather (y[p] = x[perm[p]]) or scatter (y[perm[p]] = x[p]) inside
// each (batch, head) slab; blockIdx.y is the slab.  Rows move as 16-byte
// vectors: each thread takes kPermUnroll vectors kPermThreads apart (so a
// warp's accesses stay contiguous within a row), reads all their table
// entries, then all their sources, then writes, so that every thread keeps
// kPermUnroll loads in flight against HBM.  Table entries outside [0, N) are
// skipped.  I is the index type inside a slab (32-bit whenever N * vpr fits).
constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

template <typename I>
__global__ void __launch_bounds__(kPermThreads) permute_kernel(
    const uint4* __restrict__ x, uint4* __restrict__ y, int32_t N, int32_t vpr,
    const int32_t* __restrict__ perm, int inverse) {
  const int64_t slab = int64_t(blockIdx.y) * N * vpr;
  const uint4* __restrict__ xs = x + slab;
  uint4* __restrict__ ys = y + slab;
  const I total = I(N) * I(vpr);
  const I base = I(blockIdx.x) * I(kPermThreads * kPermUnroll) + I(threadIdx.x);
  I row[kPermUnroll], col[kPermUnroll];
  int32_t q[kPermUnroll];
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    const I e = base + I(u) * I(kPermThreads);
    row[u] = e / I(vpr);
    col[u] = e - row[u] * I(vpr);
    q[u] = e < total ? __ldg(perm + row[u]) : -1;
  }
  uint4 val[kPermUnroll];
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    if (uint32_t(q[u]) < uint32_t(N)) {
      const I src = inverse ? row[u] : I(q[u]);
      val[u] = __ldg(xs + src * I(vpr) + col[u]);
    }
  }
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    if (uint32_t(q[u]) < uint32_t(N)) {
      const I dst = inverse ? I(q[u]) : row[u];
      ys[dst * I(vpr) + col[u]] = val[u];
    }
  }
}

bool make_grid(int32_t T, int32_t Hg, int32_t Wg, HilbertGrid* g) {
  const int32_t ext[3] = {T, Hg, Wg};
  const int32_t mul[3] = {Hg * Wg, Wg, 1};
  g->n = 0;
  int32_t mx = 1;
  for (int a = 0; a < 3; ++a) {
    if (ext[a] > 1) {
      g->ext[g->n] = ext[a];
      g->mul[g->n] = mul[a];
      ++g->n;
      if (ext[a] > mx) mx = ext[a];
    }
  }
  g->bits = 0;
  while ((1 << g->bits) < mx) ++g->bits;
  if (g->bits == 0) g->bits = 1;
  if (g->n * g->bits > 30) return false;
  g->cube = g->n == 0 ? 0 : (int64_t(1) << (g->n * g->bits));
  return true;
}

}  // namespace

size_t hilbert_ws_bytes(int32_t T, int32_t Hg, int32_t Wg) {
  HilbertGrid g;
  if (T < 1 || Hg < 1 || Wg < 1 || !make_grid(T, Hg, Wg, &g)) return 0;
  return align256(size_t(cdiv(g.cube, kHilPerCta) + 1) * sizeof(int32_t));
}

cudaError_t launch_hilbert_index(int32_t N, int32_t prefix_len, int32_t T, int32_t Hg,
                                 int32_t Wg, int32_t* perm, void* ws, cudaStream_t s) {
  HilbertGrid g;
  if (!make_grid(T, Hg, Wg, &g)) return cudaErrorInvalidValue;
  const int32_t L = T * Hg * Wg;
  int32_t* counts = static_cast<int32_t*>(ws);
  // a grid without an axis of extent > 1 has cube 0: the table is the identity
  const int64_t ctas = g.cube > 0 ? cdiv(g.cube, kHilPerCta) : 0;
  const int64_t fill_ctas = cdiv(N, kHilThreads);
  int64_t grid = ctas > fill_ctas ? ctas : fill_ctas;
  if (grid < 1) grid = 1;
  const int32_t Lg = g.cube > 0 ? L : 0;
  auto run = [&](auto na) -> cudaError_t {
    constexpr int NA = decltype(na)::value;
    if (ctas > 0) {
      hilbert_count_kernel<NA><<<unsigned(ctas), kHilThreads, 0, s>>>(g, counts);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    hilbert_scatter_kernel<NA><<<unsigned(grid), kHilThreads, 0, s>>>(
        g, counts, int32_t(ctas), N, prefix_len, Lg, perm);
    return cudaGetLastError();
  };
  // a grid without an axis of extent > 1 launches no decode (cube 0)
  if (g.n == 3) return run(std::integral_constant<int, 3>{});
  if (g.n == 2) return run(std::integral_constant<int, 2>{});
  return run(std::integral_constant<int, 1>{});
}

cudaError_t launch_permute_rows(const void* x, void* y, int64_t BH, int32_t N, int32_t row_bytes,
                                const int32_t* perm, bool inverse, cudaStream_t s) {
  const int32_t vpr = row_bytes / 16;
  const int64_t total = int64_t(N) * vpr;
  const int64_t gx = cdiv(total, int64_t(kPermThreads) * kPermUnroll);
  if (gx < 1 || gx > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid{unsigned(gx), unsigned(BH), 1u};
  const auto* xs = static_cast<const uint4*>(x);
  auto* ys = static_cast<uint4*>(y);
  // the last thread's index, base + (kPermUnroll - 1) * kPermThreads, stays
  // below gx * kPermThreads * kPermUnroll <= total + kPermThreads * kPermUnroll
  if (total + int64_t(kPermThreads) * kPermUnroll <= 0x7fffffffLL)
    permute_kernel<int32_t><<<grid, kPermThreads, 0, s>>>(xs, ys, N, vpr, perm, inverse ? 1 : 0);
  else
    permute_kernel<int64_t><<<grid, kPermThreads, 0, s>>>(xs, ys, N, vpr, perm, inverse ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sparge
