// Tensor Cache second tier ("Tensor Cache: Eviction-conditioned Associative
// Memory for Transformers", section "Metodología"): the hot ring is the
// first level; every token it displaces is written into a d x d
// outer-product matrix A per (row, kv head) ("Mecanismo de Escritura"), and
// a query reads A back as q A ("Mecanismo de Lectura"), added to the ring's
// softmax output through a sigmoid gate ("Fusión").
//
//   tc_update  one block per (unit, 16 rows of A), one thread per column.
//              A run of E evictions is applied in one pass as the weighted
//              sum the page's parallel scan computes (lambda^E A plus
//              eta lambda^(E-1-e) k_e v_e^T), equal to E sequential writes.
//              Algorithmic bytes per unit: 8 d^2 (A read and written) plus
//              4 d per evicted token.
//   tc_read    one block per unit: 4 row groups x one thread per column,
//              each thread loading its 1/4 column of A at once; every
//              element of A is read once and multiplied by all G query heads
//              of the unit, and the row groups' sums meet in shared memory.
//              4 d^2 bytes per unit.
#include <cmath>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr int kTcRows = 16;          // rows of A per update block
constexpr int kTcBatch = 32;         // evicted tokens staged per pass
constexpr int kTcMaxGroup = 8;
constexpr int kTcReadSplit = 4;      // row groups of A per read block (threads = d x 4)

template <int D>
__global__ void __launch_bounds__(D) tc_update_kernel(const TcUpdateArgs a) {
  __shared__ float ks[kTcBatch][kTcRows];
  __shared__ float wsh[kTcBatch];
  constexpr int BPU = D / kTcRows;                  // blocks per unit
  const int unit = blockIdx.x / BPU, i0 = (blockIdx.x % BPU) * kTcRows;
  const int j = threadIdx.x;
  const int kvh = unit % a.Hkv;
  const double lam = a.lam[kvh], eta = a.eta[kvh];
  const int E = a.nA + a.nB;
  auto token = [&](const __half* ring, const __half* src, int e) {
    if (e < a.nA) {
      int slot = a.ring_start + e;
      if (slot >= a.W) slot -= a.W;
      return ring + ((size_t)unit * a.W + slot) * D;
    }
    return src + ((size_t)unit * a.src_tokens + (e - a.nA)) * D;
  };
  float* Au = a.A + (size_t)unit * D * D;
  const float decay = (float)pow(lam, (double)E);
  float acc[kTcRows];
#pragma unroll
  for (int r = 0; r < kTcRows; ++r) acc[r] = decay * Au[(size_t)(i0 + r) * D + j];
  for (int e0 = 0; e0 < E; e0 += kTcBatch) {
    const int nb = E - e0 < kTcBatch ? E - e0 : kTcBatch;
    __syncthreads();
    for (int x = j; x < nb * kTcRows; x += D) {
      const int e = x / kTcRows, r = x % kTcRows;
      ks[e][r] = __half2float(token(a.ring_k, a.src_k, e0 + e)[i0 + r]);
    }
    if (j < nb) wsh[j] = (float)(eta * pow(lam, (double)(E - 1 - (e0 + j))));
    __syncthreads();
    for (int e = 0; e < nb; ++e) {
      const float vj = wsh[e] * __half2float(token(a.ring_v, a.src_v, e0 + e)[j]);
#pragma unroll
      for (int r = 0; r < kTcRows; ++r) acc[r] = fmaf(ks[e][r], vj, acc[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < kTcRows; ++r) Au[(size_t)(i0 + r) * D + j] = acc[r];
}

template <int D>
__global__ void __launch_bounds__(D * kTcReadSplit) tc_read_kernel(const TcReadArgs a) {
  constexpr int R = D / kTcReadSplit;               // rows of A per thread
  __shared__ float qs[kTcMaxGroup][D];
  __shared__ float part[kTcReadSplit - 1][kTcMaxGroup][D];
  const int unit = blockIdx.x, t = threadIdx.x;
  const int col = t % D, grp = t / D;               // column, and row group of R rows
  const int head0 = unit * a.G;                     // b * Hq + kvh * G
  for (int x = t; x < a.G * D; x += D * kTcReadSplit)
    qs[x / D][x % D] = __half2float(a.q[(size_t)head0 * D + x]);
  const float* Au = a.A + (size_t)unit * D * D + (size_t)grp * R * D + col;
  float av[R];
#pragma unroll
  for (int i = 0; i < R; ++i) av[i] = Au[(size_t)i * D];   // every load before any use
  __syncthreads();
  float m[kTcMaxGroup];
#pragma unroll
  for (int g = 0; g < kTcMaxGroup; ++g) {
    m[g] = 0.f;
    if (g < a.G) {
#pragma unroll
      for (int i = 0; i < R; ++i) m[g] = fmaf(qs[g][grp * R + i], av[i], m[g]);
    }
  }
  if (grp > 0) {
#pragma unroll
    for (int g = 0; g < kTcMaxGroup; ++g)
      if (g < a.G) part[grp - 1][g][col] = m[g];
  }
  __syncthreads();
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < kTcMaxGroup; ++g) {
      if (g < a.G) {
        float sum = m[g];
#pragma unroll
        for (int r = 0; r < kTcReadSplit - 1; ++r) sum += part[r][g][col];
        const int h = head0 + g;
        a.out[(size_t)h * D + col] += a.sig[h % a.Hq] * sum;
      }
    }
  }
}

}  // namespace

cudaError_t launch_tc_update(const TcUpdateArgs& a, cudaStream_t s) {
  if (a.nA + a.nB <= 0) return cudaSuccess;
  if (a.d == 64)
    tc_update_kernel<64><<<a.units * (64 / kTcRows), 64, 0, s>>>(a);
  else if (a.d == 128)
    tc_update_kernel<128><<<a.units * (128 / kTcRows), 128, 0, s>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_tc_read(const TcReadArgs& a, cudaStream_t s) {
  if (a.G > kTcMaxGroup) return cudaErrorInvalidValue;
  if (a.d == 64)
    tc_read_kernel<64><<<a.units, 64 * kTcReadSplit, 0, s>>>(a);
  else if (a.d == 128)
    tc_read_kernel<128><<<a.units, 128 * kTcReadSplit, 0, s>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace tq
