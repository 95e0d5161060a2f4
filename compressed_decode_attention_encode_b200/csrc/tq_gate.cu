// Threshold gate of the cold tier for gated decode calls ("Monarch v3 ...",
// "Bucle de Decodificación Simplificado": the hot scores come first, and the
// cold pages are read only while the largest hot score is below a
// threshold).  Writes the per-head decisions and the list of (row, kv head)
// units whose cold tier the attention kernel still streams.
#include <cfloat>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// Blocks of 256 threads; block (unit, c) takes rows [c * ROWS, (c + 1) *
// ROWS) of the unit's hot window.  A hot K row is read as D/8 lanes x 16
// bytes, so one warp load covers 32/(D/8) rows, and each lane issues all
// kGateUnroll of its loads before it computes.  Per row and query head a
// lane multiplies its 8 coordinates and a butterfly over the row's lanes
// gives q.k.
// The gate is a programmatic dependent of q-prep, so it starts while the
// step's eviction and q-prep still run.  Before it waits for them it reads
// only what they do not write (the queries, and the ring rows other than
// the last eviction's slots); the evicted-into rows come after the wait.
// When the last eviction wrote more than kGateEarlyRows slots, the whole
// window is read after the wait.
// The block stores its per-head maxima in its own cmax slot;
// the block that finishes last reduces each head's slots (all loads issued
// at once), takes the decisions, lists the units that still read their
// cold tier and leaves the counter at 0 for the next call.
// ---------------------------------------------------------------------------
constexpr int kGateThreads = 256;
constexpr int kGateMaxGroup = 8;
constexpr int kGateUnroll = 8;
constexpr int kGateEarlyRows = 8;

template <int D>
struct GateShape {
  static constexpr int LPR = D / 8;                 // lanes per row (16 bytes each)
  static constexpr int RPI = 32 / LPR;              // rows per warp load
  static constexpr int NW = kGateThreads / 32;
  static constexpr int ROWS = NW * RPI * kGateUnroll;   // rows per block
};

static_assert(GateShape<128>::ROWS == kGateRowsMin && GateShape<64>::ROWS >= kGateRowsMin,
              "gate blocks take at least kGateRowsMin rows (sizes the cmax slots)");

template <int D>
__global__ void __launch_bounds__(kGateThreads) gate_kernel(const GateArgs a) {
  using S = GateShape<D>;
  constexpr int LPR = S::LPR, RPI = S::RPI, NW = S::NW;
  __shared__ float wmax[NW][kGateMaxGroup];
  __shared__ int wcnt[NW];
  __shared__ int is_last;
  const int chunks = gridDim.x / a.units;
  const int unit = blockIdx.x / chunks, chunk = blockIdx.x % chunks, r0 = chunk * S::ROWS;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int head0 = (unit / a.Hkv) * a.Hq + (unit % a.Hkv) * a.G;
  const int col = (lane % LPR) * 8;                 // this lane's 8 coordinates
  const int sub = lane / LPR;                       // its row within a warp load
  const bool early = a.dirty_n <= kGateEarlyRows;
  auto dirty = [&](int r) {
    int o = r - a.dirty_lo;
    if (o < 0) o += a.W;
    return o < a.dirty_n;
  };
  float qr[kGateMaxGroup][8], mx[kGateMaxGroup];
#pragma unroll
  for (int g = 0; g < kGateMaxGroup; ++g) mx[g] = -INFINITY;
  // q.k of one 16-byte slice per lane, summed over the row's lanes; rows
  // with ok == false leave the maxima alone
  auto fold_row = [&](const uint4& w, bool ok) {
    float kf[8];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
      kf[2 * e] = f.x;
      kf[2 * e + 1] = f.y;
    }
#pragma unroll
    for (int g = 0; g < kGateMaxGroup; ++g) {
      if (g < a.G) {
        float sc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) sc = fmaf(qr[g][e], kf[e], sc);
#pragma unroll
        for (int o = LPR / 2; o; o >>= 1) sc += __shfl_xor_sync(kFull, sc, o);
        if (ok) mx[g] = fmaxf(mx[g], sc);
      }
    }
  };
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
  // the window's loads first ...
  const __half* kbase = a.hot_k + (size_t)unit * a.W * D + col;
  uint4 kw[kGateUnroll];
  bool ok[kGateUnroll];
#pragma unroll
  for (int u = 0; u < kGateUnroll; ++u) {
    const int row = r0 + (u * NW + warp) * RPI + sub;
    ok[u] = row < a.n_hot && !(early && dirty(row));
    kw[u] = ok[u] ? __ldg(reinterpret_cast<const uint4*>(kbase + (size_t)row * D))
                  : make_uint4(0u, 0u, 0u, 0u);
  }
  // ... then the queries
#pragma unroll
  for (int g = 0; g < kGateMaxGroup; ++g) {
    if (g < a.G) {
      const uint4 w = *reinterpret_cast<const uint4*>(a.q + (size_t)(head0 + g) * D + col);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
        qr[g][2 * e] = f.x;
        qr[g][2 * e + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qr[g][e] = 0.f;
    }
  }
#pragma unroll
  for (int u = 0; u < kGateUnroll; ++u) fold_row(kw[u], ok[u]);
  if (early) {
    // the last eviction's rows, once the eviction and q-prep have finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int j = warp; j < a.dirty_n; j += NW) {
      int slot = a.dirty_lo + j;
      if (slot >= a.W) slot -= a.W;
      if (slot < r0 || slot >= r0 + S::ROWS || slot >= a.n_hot) continue;   // warp-uniform
      const bool mine = sub == 0;          // the first row-group of lanes reads it
      const uint4 w = mine ? __ldcg(reinterpret_cast<const uint4*>(kbase + (size_t)slot * D))
                           : make_uint4(0u, 0u, 0u, 0u);
      fold_row(w, mine);
    }
  }
#pragma unroll
  for (int g = 0; g < kGateMaxGroup; ++g)
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(kFull, mx[g], o));
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < kGateMaxGroup; ++g) wmax[warp][g] = mx[g];
  }
  __syncthreads();
  if (t < a.G) {
    float m = wmax[0][t];
    for (int w = 1; w < NW; ++w) m = fmaxf(m, wmax[w][t]);
    a.cmax[(size_t)(head0 + t) * chunks + chunk] = m;
    __threadfence();              // the slot is visible before this block counts itself done
  }
  __syncthreads();
  if (t == 0) {
    __threadfence();
    is_last = atomicAdd(a.counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last) return;
  // ---- last block: decisions, then the active units in unit order -------
  __threadfence();
  int base = 0;
  for (int u0 = 0; u0 < a.units; u0 += kGateThreads) {
    const int u = u0 + t;
    int act = 0;
    if (u < a.units) {
      const int h0 = (u / a.Hkv) * a.Hq + (u % a.Hkv) * a.G;
      float m[kGateMaxGroup];
#pragma unroll
      for (int g = 0; g < kGateMaxGroup; ++g) m[g] = -INFINITY;
      for (int c0 = 0; c0 < chunks; c0 += 4) {
        float v[4][kGateMaxGroup];                   // every read issued before any is used
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int g = 0; g < kGateMaxGroup; ++g)    // L2 reads: written by other blocks
            v[cc][g] = (g < a.G && c0 + cc < chunks)
                           ? __ldcg(a.cmax + (size_t)(h0 + g) * chunks + c0 + cc) : -INFINITY;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int g = 0; g < kGateMaxGroup; ++g) m[g] = fmaxf(m[g], v[cc][g]);
      }
#pragma unroll
      for (int g = 0; g < kGateMaxGroup; ++g) {
        if (g < a.G) {
          const int skip = (a.n_hot > 0 && m[g] >= a.threshold) ? 1 : 0;
          a.head_skip[h0 + g] = skip;
          act |= !skip;
        }
      }
    }
    const unsigned bal = __ballot_sync(kFull, act);
    if (lane == 0) wcnt[warp] = __popc(bal);
    __syncthreads();
    int off = base, tot = 0;
    for (int w = 0; w < NW; ++w) {
      if (w < warp) off += wcnt[w];
      tot += wcnt[w];
    }
    if (u < a.units) {
      const int p = off + __popc(bal & ((1u << lane) - 1u));
      a.unit_pos[u] = act ? p : -1;
      if (act) a.alist[p] = u;
    }
    base += tot;
    __syncthreads();
  }
  for (int p = base + t; p <= a.units; p += kGateThreads) a.alist[p] = 0;
  if (t == 0) {
    *a.n_active = base;
    *a.counter = 0u;
  }
}

}  // namespace

template <int D>
cudaError_t launch_gate_d(const GateArgs& a, cudaStream_t s) {
  const int chunks = a.n_hot > 0 ? (a.n_hot + GateShape<D>::ROWS - 1) / GateShape<D>::ROWS : 1;
  // programmatic dependent of q-prep (which lets dependents start at once)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.units * chunks);
  cfg.blockDim = dim3(kGateThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gate_kernel<D>, a);
}

cudaError_t launch_gate(const GateArgs& a, cudaStream_t s) {
  if (a.G > kGateMaxGroup) return cudaErrorInvalidValue;
  if (a.d == 64) return launch_gate_d<64>(a, s);
  if (a.d == 128) return launch_gate_d<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace tq
