// The float64 per-vector encode shared by the KV-cache encoder and the
// vector-search encoder: randomized Hadamard rotation, polar codes with an
// fp16 scale, and (for keys) the QJL sign sketch of the residual.
#pragma once

#include "tq_internal.cuh"

namespace tq {
namespace enc {

constexpr unsigned kFull = 0xffffffffu;
constexpr double kTwoPi = 6.283185307179586476925286766559;  // rounds to 2 * fp64(pi)
constexpr int kMaxSignWords = 8;   // m <= 256 sign bits per vector

__device__ __forceinline__ uint16_t f64_to_f16_bits(double x) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
  return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
}

// Angle tables (nt = 2^b_theta codes), built on the host when a handle is
// created (angle_table_host) and copied into a block's shared memory by
// angle_tables before its first encode:
//   bnd[0]      (cos, sin)(pi / nt): the half-sector rotation
//   bnd[1 + j]  (cos, sin)(2 pi (j + 1) / nt), j < nt/4 - 1: the sector
//               boundaries inside the first quadrant
//   cs[c]       (cos, sin)(c 2 pi / nt), at angle_cs_offset(nt) + c: the
//               dequantized directions of the residual step
__device__ __forceinline__ void angle_tables(int nt, const double2* src, double2* tab, int tid, int nthreads) {
  for (int e = tid; e < angle_cs_offset(nt) + nt; e += nthreads) tab[e] = src[e];
}

// The angle code of (x, y): the nearest of the nt directions c 2 pi / nt,
// i.e. floor(theta nt / (2 pi) + 1/2) mod nt for theta = atan2(y, x).  The
// pair is rotated by half a sector, its quadrant read off the signs, and its
// sector inside the quadrant found by cross products with the boundary
// directions; rounding moves a decision only for pairs within about 1e-15
// of a sector boundary (the origin gets code 0, as atan2(0, 0) = 0 does).
__device__ __forceinline__ int angle_code(double x, double y, int nt, const double2* bnd) {
  const double2 r = bnd[0];
  const double xr = fma(x, r.x, -__dmul_rn(y, r.y));
  const double yr = fma(x, r.y, __dmul_rn(y, r.x));
  int q;
  double u, v;                               // the pair turned into the first quadrant
  if (yr >= 0.0 && xr > 0.0) { q = 0; u = xr; v = yr; }
  else if (yr > 0.0) { q = 1; u = yr; v = -xr; }
  else if (xr < 0.0) { q = 2; u = -xr; v = -yr; }
  else if (yr < 0.0) { q = 3; u = -yr; v = xr; }
  else return 0;                             // the origin
  if (nt == 2) return q >> 1;
  const int per = nt >> 2;                   // sectors per quadrant
  int j = 0;
  while (j < per - 1 && fma(bnd[1 + j].x, v, -__dmul_rn(bnd[1 + j].y, u)) >= 0.0) ++j;
  return (q * per + j) & (nt - 1);
}

template <int E>
__device__ __forceinline__ void load_vec(const __half* p, int lane, double (&x)[E]) {
  const __half* q = p + lane * E;
  if constexpr (E == 2) {
    const __half2 v = *reinterpret_cast<const __half2*>(q);
    x[0] = (double)__low2float(v);
    x[1] = (double)__high2float(v);
  } else if constexpr (E == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(q);
    const __half2 a = *reinterpret_cast<const __half2*>(&v.x);
    const __half2 b = *reinterpret_cast<const __half2*>(&v.y);
    x[0] = (double)__low2float(a); x[1] = (double)__high2float(a);
    x[2] = (double)__low2float(b); x[3] = (double)__high2float(b);
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = (double)__half2float(q[i]);
  }
}

// Encodes one vector (K or V) held at `src` in float64; writes its code
// words into `codes[0..D/2)` (shared memory, one byte per pair) and, for
// keys, its sign words into `bits` (canonical order, bit i of word i/32)
// and the raw fp16 scalars.  Whole warp; returns nothing else.
// `load(lane, x)` fills the lane's D/32 consecutive input elements (padded
// coordinates read as 0).  `L` supplies b_r, b_theta and m; `St` is S^T
// [D, m] (global or shared memory); `signs` the rotation diagonal; `atab`
// the block's angle tables (angle_tables).  With
// SKETCH false a key stops after its residual (left in rbuf[0..D)) and its
// norm; qjl_sketch_block then forms the sign words of several keys at once.
template <int D, bool SKETCH = true, typename Loader>
__device__ __forceinline__ void encode_vector_any(const Layout& L, const double* signs,
                                                  const float* St, const double2* atab,
                                                  double inv_sqrt_d, int* status,
                                                  Loader load, bool is_key, double* rbuf,
                                                  uint8_t* codes, uint32_t* bits,
                                                  uint16_t* s16_out, uint16_t* rn16_out) {
  constexpr int E = D / 32;      // elements per lane
  constexpr int PL = E / 2;      // pairs per lane
  const int lane = threadIdx.x & 31;
  const int Lr = (1 << L.b_r) - 1;
  const int nt = 1 << L.b_theta;

  // ---- rotation: y = H (D x) / sqrt(d) ----------------------------------
  double x[E];
  load(lane, x);
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = __dmul_rn(x[i], signs[lane * E + i]);
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    if (h < E) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if (!(i & h)) {
          const double p = x[i], q = x[i + h];
          x[i] = __dadd_rn(p, q);
          x[i + h] = __dsub_rn(p, q);
        }
      }
    } else {
      const int lm = h / E;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const double o = __shfl_xor_sync(kFull, x[i], lm);
        x[i] = (lane & lm) ? __dsub_rn(o, x[i]) : __dadd_rn(x[i], o);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = __dmul_rn(x[i], inv_sqrt_d);

  // ---- polar: rho and the angle code per pair; scale s16 = fp16(max rho) --
  double rho[PL];
  int ct[PL];
  double smax = 0.0;
#pragma unroll
  for (int k = 0; k < PL; ++k) {
    const double y0 = x[2 * k], y1 = x[2 * k + 1];
    rho[k] = __dsqrt_rn(__dadd_rn(__dmul_rn(y0, y0), __dmul_rn(y1, y1)));
    ct[k] = angle_code(y0, y1, nt, atab);
    smax = fmax(smax, rho[k]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) smax = fmax(smax, __shfl_xor_sync(kFull, smax, o));
  uint16_t s16b = f64_to_f16_bits(smax);
  if ((s16b & 0x7c00u) == 0x7c00u) {       // overflow: latch, store a zero record
    if (lane == 0) atomicOr(status, kStatusRange);
    s16b = 0;
  }
  const double s16 = f16_bits_to_f64(s16b);
  const bool zero = (s16 == 0.0);

  // ---- codes ---------------------------------------------------------------
  int cr[PL];
#pragma unroll
  for (int k = 0; k < PL; ++k) {
    const double tr = __dmul_rn(__ddiv_rn(rho[k], zero ? 1.0 : s16), (double)Lr);
    const int c = (int)rint(tr);
    cr[k] = c < 0 ? 0 : (c > Lr ? Lr : c);
    if (zero) { cr[k] = 0; ct[k] = 0; }
    codes[lane * PL + k] = (uint8_t)((cr[k] << L.b_theta) | ct[k]);
  }
  if (lane == 0) *s16_out = s16b;

  // ---- residual and QJL sketch (keys) -------------------------------------
  if (is_key) {
    double r[E];
    double ss = 0.0;
#pragma unroll
    for (int k = 0; k < PL; ++k) {
      const double rh = __ddiv_rn(__dmul_rn((double)cr[k], s16), (double)Lr);
      const double2 csn = atab[angle_cs_offset(nt) + ct[k]];   // cos, sin of c_theta 2 pi / nt
      r[2 * k] = __dsub_rn(x[2 * k], __dmul_rn(rh, csn.x));
      r[2 * k + 1] = __dsub_rn(x[2 * k + 1], __dmul_rn(rh, csn.y));
      ss = __dadd_rn(ss, __dadd_rn(__dmul_rn(r[2 * k], r[2 * k]), __dmul_rn(r[2 * k + 1], r[2 * k + 1])));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
    const uint16_t rnb = f64_to_f16_bits(__dsqrt_rn(ss));
    if ((rnb & 0x7c00u) == 0x7c00u && lane == 0) atomicOr(status, kStatusRange);
    if (lane == 0) *rn16_out = rnb;
#pragma unroll
    for (int i = 0; i < E; ++i) rbuf[lane * E + i] = r[i];
    __syncwarp();
    if constexpr (!SKETCH) return;
    // (S r)_i for the lane's outputs i = lane + 32 k, all k at once so that
    // the loads of a batch of rows of S^T are in flight together; each
    // output still sums over j in ascending order.
    const int m = L.m;
    const int nk = (m + 31) >> 5;
    double acc[kMaxSignWords];
#pragma unroll
    for (int k = 0; k < kMaxSignWords; ++k) acc[k] = 0.0;
    constexpr int JB = 4;
    for (int j0 = 0; j0 < D; j0 += JB) {
      float sv[JB][kMaxSignWords];
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) {
#pragma unroll
        for (int k = 0; k < kMaxSignWords; ++k) {
          const int i = lane + 32 * k;
          sv[jj][k] = (k < nk && i < m) ? St[(size_t)(j0 + jj) * m + i] : 0.f;
        }
      }
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) {
        const double rj = rbuf[j0 + jj];
#pragma unroll
        for (int k = 0; k < kMaxSignWords; ++k)
          if (k < nk) acc[k] = fma((double)sv[jj][k], rj, acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxSignWords; ++k) {
      if (k < nk) {
        const unsigned word = __ballot_sync(kFull, lane + 32 * k < m && acc[k] >= 0.0);
        if (lane == 0) bits[k] = word;
      }
    }
  }
  __syncwarp();
}

// A key and a value of one token at once (whole warp; the bulk encode):
// the steps of encode_vector_any for the two vectors, interleaved stage by
// stage so that every stage has two independent float64 chains.  Each
// vector sees exactly the operations encode_vector_any applies to it, so
// the codes are the same.  The key stops after its residual (kept in rbuf
// for a sketch blocked over keys).
template <int D>
__device__ __forceinline__ void encode_kv_pair(const Layout& L, const double* signs, const double2* atab,
                                               double inv_sqrt_d, int* status, const __half* ksrc,
                                               const __half* vsrc, double* rbuf, uint8_t* kcodes,
                                               uint8_t* vcodes, uint16_t* ks16_out, uint16_t* rn16_out,
                                               uint16_t* vs16_out) {
  constexpr int E = D / 32;      // elements per lane
  constexpr int PL = E / 2;      // pairs per lane
  const int lane = threadIdx.x & 31;
  const int Lr = (1 << L.b_r) - 1;
  const int nt = 1 << L.b_theta;

  // ---- rotation: y = H (D x) / sqrt(d), key (v = 0) and value (v = 1) ------
  double x[2][E];
  load_vec<E>(ksrc, lane, x[0]);
  load_vec<E>(vsrc, lane, x[1]);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const double sg = signs[lane * E + i];
    x[0][i] = __dmul_rn(x[0][i], sg);
    x[1][i] = __dmul_rn(x[1][i], sg);
  }
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    if (h < E) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if (!(i & h)) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const double p = x[v][i], q = x[v][i + h];
            x[v][i] = __dadd_rn(p, q);
            x[v][i + h] = __dsub_rn(p, q);
          }
        }
      }
    } else {
      const int lm = h / E;
#pragma unroll
      for (int i = 0; i < E; ++i) {
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const double o = __shfl_xor_sync(kFull, x[v][i], lm);
          x[v][i] = (lane & lm) ? __dsub_rn(o, x[v][i]) : __dadd_rn(x[v][i], o);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < E; ++i) {
    x[0][i] = __dmul_rn(x[0][i], inv_sqrt_d);
    x[1][i] = __dmul_rn(x[1][i], inv_sqrt_d);
  }

  // ---- polar: rho and the angle code per pair; scale s16 = fp16(max rho) --
  double rho[2][PL];
  int ct[2][PL];
  double smax[2] = {0.0, 0.0};
#pragma unroll
  for (int k = 0; k < PL; ++k) {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const double y0 = x[v][2 * k], y1 = x[v][2 * k + 1];
      rho[v][k] = __dsqrt_rn(__dadd_rn(__dmul_rn(y0, y0), __dmul_rn(y1, y1)));
      ct[v][k] = angle_code(y0, y1, nt, atab);
      smax[v] = fmax(smax[v], rho[v][k]);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    smax[0] = fmax(smax[0], __shfl_xor_sync(kFull, smax[0], o));
    smax[1] = fmax(smax[1], __shfl_xor_sync(kFull, smax[1], o));
  }
  uint16_t s16b[2];
  double s16[2];
  bool zero[2];
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    s16b[v] = f64_to_f16_bits(smax[v]);
    if ((s16b[v] & 0x7c00u) == 0x7c00u) {   // overflow: latch, store a zero record
      if (lane == 0) atomicOr(status, kStatusRange);
      s16b[v] = 0;
    }
    s16[v] = f16_bits_to_f64(s16b[v]);
    zero[v] = (s16[v] == 0.0);
  }

  // ---- codes ---------------------------------------------------------------
  int cr[2][PL];
#pragma unroll
  for (int k = 0; k < PL; ++k) {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const double tr = __dmul_rn(__ddiv_rn(rho[v][k], zero[v] ? 1.0 : s16[v]), (double)Lr);
      const int c = (int)rint(tr);
      cr[v][k] = c < 0 ? 0 : (c > Lr ? Lr : c);
      if (zero[v]) {
        cr[v][k] = 0;
        ct[v][k] = 0;
      }
    }
    kcodes[lane * PL + k] = (uint8_t)((cr[0][k] << L.b_theta) | ct[0][k]);
    vcodes[lane * PL + k] = (uint8_t)((cr[1][k] << L.b_theta) | ct[1][k]);
  }
  if (lane == 0) {
    *ks16_out = s16b[0];
    *vs16_out = s16b[1];
  }

  // ---- the key's residual r = y - y_hat and its norm rn16 -----------------
  double r[E];
  double ss = 0.0;
#pragma unroll
  for (int k = 0; k < PL; ++k) {
    const double rh = __ddiv_rn(__dmul_rn((double)cr[0][k], s16[0]), (double)Lr);
    const double2 csn = atab[angle_cs_offset(nt) + ct[0][k]];   // cos, sin of c_theta 2 pi / nt
    r[2 * k] = __dsub_rn(x[0][2 * k], __dmul_rn(rh, csn.x));
    r[2 * k + 1] = __dsub_rn(x[0][2 * k + 1], __dmul_rn(rh, csn.y));
    ss = __dadd_rn(ss, __dadd_rn(__dmul_rn(r[2 * k], r[2 * k]), __dmul_rn(r[2 * k + 1], r[2 * k + 1])));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
  const uint16_t rnb = f64_to_f16_bits(__dsqrt_rn(ss));
  if ((rnb & 0x7c00u) == 0x7c00u && lane == 0) atomicOr(status, kStatusRange);
  if (lane == 0) *rn16_out = rnb;
#pragma unroll
  for (int i = 0; i < E; ++i) rbuf[lane * E + i] = r[i];
  __syncwarp();
}

// QJL sign words of NV residuals at once (whole warp): r_v = rbuf[v D ..
// v D + D), words written to bits[v * bits_stride + k] for the vectors with
// live[v].  Lane outputs i = lane + 32 k as in encode_vector_any; each S^T
// value is loaded and widened once and feeds NV fp64 FMAs, and each output
// still sums over j in ascending order (the same FMAs as one vector alone).
// MC: m when known at compile time (0: the run-time m).
template <int D, int NV, int NK, int MC = 0>
__device__ __forceinline__ void qjl_sketch_block(int m_rt, const float* St, const double* rbuf,
                                                 const bool (&live)[NV], uint32_t* bits, int bits_stride) {
  const int m = MC ? MC : m_rt;
  const int lane = threadIdx.x & 31;
  double acc[NV][NK];
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int k = 0; k < NK; ++k) acc[v][k] = 0.0;
  constexpr int JB = 2;
  for (int j0 = 0; j0 < D; j0 += JB) {
    double sv[JB][NK];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj)
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        const int i = lane + 32 * k;
        sv[jj][k] = i < m ? (double)St[(size_t)(j0 + jj) * m + i] : 0.0;
      }
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const double rj = rbuf[v * D + j0 + jj];
#pragma unroll
        for (int k = 0; k < NK; ++k) acc[v][k] = fma(sv[jj][k], rj, acc[v][k]);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
#pragma unroll
    for (int k = 0; k < NK; ++k) {
      const unsigned word = __ballot_sync(kFull, lane + 32 * k < m && acc[v][k] >= 0.0);
      if (lane == 0 && live[v] && 32 * k < m) bits[v * bits_stride + k] = word;
    }
  }
  __syncwarp();
}


// The same sign words from S^T in lane order (stl: [D][32][NK] floats in
// shared memory, element (j, l, k) = S^T[j][l + 32 k], m = 32 NK): each
// lane reads its NK values of a row with one vector load and two residual
// values of a key with one; the FMAs and their order are those of
// qjl_sketch_block.
template <int D, int NV, int NK>
__device__ __forceinline__ void qjl_sketch_lanes(const float* stl, const double* rbuf, const bool (&live)[NV],
                                                 uint32_t* bits, int bits_stride) {
  static_assert(NK == 2 || NK == 4, "m = 64 or 128");
  const int lane = threadIdx.x & 31;
  double acc[NV][NK];
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int k = 0; k < NK; ++k) acc[v][k] = 0.0;
  for (int j0 = 0; j0 < D; j0 += 2) {
    double sv[2][NK];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const float* row = stl + ((j0 + jj) * 32 + lane) * NK;
      if constexpr (NK == 4) {
        const float4 f = *reinterpret_cast<const float4*>(row);
        sv[jj][0] = (double)f.x;
        sv[jj][1] = (double)f.y;
        sv[jj][2] = (double)f.z;
        sv[jj][3] = (double)f.w;
      } else {
        const float2 f = *reinterpret_cast<const float2*>(row);
        sv[jj][0] = (double)f.x;
        sv[jj][1] = (double)f.y;
      }
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const double2 r2 = *reinterpret_cast<const double2*>(rbuf + v * D + j0);
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        acc[v][k] = fma(sv[0][k], r2.x, acc[v][k]);
        acc[v][k] = fma(sv[1][k], r2.y, acc[v][k]);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
#pragma unroll
    for (int k = 0; k < NK; ++k) {
      const unsigned word = __ballot_sync(kFull, acc[v][k] >= 0.0);
      if (lane == 0 && live[v]) bits[v * bits_stride + k] = word;
    }
  }
  __syncwarp();
}

}  // namespace enc
}  // namespace tq
