// Encode kernel: TurboQuant-style compression of K/V vectors into the cold
// store, one warp per vector.
//
// Steps ("TurboQuant: kompresja KV-cache w LLM 6 razy ...", section
// "Zasada działania PolarQuant": rotate at random, map to radius/angle,
// quantize; section "Kompensacja błędów przez QJL": 1-bit code of the
// residual), with the concrete format of this library:
//   y = H_d (D x) / sqrt(d)        Sylvester Hadamard, butterflies in
//                                  registers and across lanes (shuffles)
//   rho_j, theta_j of pair (y_2j, y_2j+1); s16 = fp16(max rho)
//   c_r = clamp(rint(rho / s16 * (2^b_r - 1)))    endpoint radius grid
//   c_th = rint(theta * 2^b_th / 2pi) mod 2^b_th  periodic angle grid
//   keys: r = y - y_hat, rn16 = fp16(||r||), bit_i = [(S r)_i >= 0]
// Every decision quantity is computed in float64 with the operations in the
// order the definition states (explicit _rn intrinsics, no contraction), so
// the codes match a float64 reference except at exact rounding ties.
#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr double kTwoPi = 6.283185307179586476925286766559;  // rounds to 2 * fp64(pi)

__device__ __forceinline__ uint16_t f64_to_f16_bits(double x) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
  return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
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

// One vector per warp.  D = padded length (power of two, >= 64).
template <int D>
__global__ void __launch_bounds__(256) encode_kernel(EncodeArgs a) {
  constexpr int E = D / 32;      // elements per lane
  constexpr int PL = E / 2;      // pairs per lane
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  extern __shared__ double smem[];
  double* rbuf = smem + warp * D;                                        // residual
  uint8_t* cbuf = reinterpret_cast<uint8_t*>(smem + warps * D) + warp * (D / 2);  // code words

  const Layout& L = a.L;
  const int Lr = (1 << L.b_r) - 1;
  const int nt = 1 << L.b_theta;
  const int bw = L.bw;
  const int m = L.m;
  const int64_t per_unit = (int64_t)a.nA + a.nB;
  const int64_t per_kind = (int64_t)a.units * per_unit;
  const int64_t jobs = 2 * per_kind;

  for (int64_t job = (int64_t)blockIdx.x * warps + warp; job < jobs;
       job += (int64_t)gridDim.x * warps) {
    const bool is_key = job < per_kind;
    const int64_t j = is_key ? job : job - per_kind;
    const int unit = (int)(j / per_unit);
    const int64_t e = j % per_unit;
    const __half* src;
    if (e < a.nA) {
      const int slot = (int)((a.ring_start + e) % a.W);
      src = (is_key ? a.ring_k : a.ring_v) + ((int64_t)unit * a.W + slot) * D;
    } else {
      src = (is_key ? a.src_k : a.src_v) + ((int64_t)unit * a.src_tokens + (e - a.nA)) * D;
    }

    // ---- rotation: y = H (D x) / sqrt(d) --------------------------------
    double x[E];
    load_vec<E>(src, lane, x);
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = __dmul_rn(x[i], a.signs[lane * E + i]);
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
    for (int i = 0; i < E; ++i) x[i] = __dmul_rn(x[i], a.inv_sqrt_d);

    // ---- polar: rho, theta per pair; scale s16 = fp16(max rho) ----------
    double rho[PL], th[PL];
    double smax = 0.0;
#pragma unroll
    for (int k = 0; k < PL; ++k) {
      const double y0 = x[2 * k], y1 = x[2 * k + 1];
      rho[k] = __dsqrt_rn(__dadd_rn(__dmul_rn(y0, y0), __dmul_rn(y1, y1)));
      th[k] = atan2(y1, y0);
      smax = fmax(smax, rho[k]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) smax = fmax(smax, __shfl_xor_sync(kFull, smax, o));
    uint16_t s16b = f64_to_f16_bits(smax);
    if ((s16b & 0x7c00u) == 0x7c00u) {       // overflow: latch, store a zero record
      if (lane == 0) atomicOr(a.status, kStatusRange);
      s16b = 0;
    }
    const double s16 = f16_bits_to_f64(s16b);
    const bool zero = (s16 == 0.0);

    // ---- codes ---------------------------------------------------------
    int cr[PL], ct[PL];
#pragma unroll
    for (int k = 0; k < PL; ++k) {
      const double tr = __dmul_rn(__ddiv_rn(rho[k], zero ? 1.0 : s16), (double)Lr);
      int c = (int)rint(tr);
      cr[k] = c < 0 ? 0 : (c > Lr ? Lr : c);
      const double tt = __ddiv_rn(__dmul_rn(th[k], (double)nt), kTwoPi);
      ct[k] = ((int)rint(tt)) & (nt - 1);
      if (zero) { cr[k] = 0; ct[k] = 0; }
      cbuf[lane * PL + k] = (uint8_t)((cr[k] << L.b_theta) | ct[k]);
    }

    const int64_t t = a.cold_start + e;
    uint8_t* blk = a.cold + ((int64_t)unit * L.blocks_per_unit + t / kTokensPerBlock) * L.block_bytes;
    const int row = (int)(t % kTokensPerBlock);
    uint8_t* rec_codes = blk + (is_key ? L.off_kc : L.off_vc) + row * L.kc_bytes;
    uint16_t* rec_scale = reinterpret_cast<uint16_t*>(blk + (is_key ? L.off_ksc : L.off_vsc)) + row;

    // ---- residual and QJL sketch (keys) ---------------------------------
    if (is_key) {
      double r[E];
      double ss = 0.0;
#pragma unroll
      for (int k = 0; k < PL; ++k) {
        const double rh = __ddiv_rn(__dmul_rn((double)cr[k], s16), (double)Lr);
        const double ang = __ddiv_rn(__dmul_rn((double)ct[k], kTwoPi), (double)nt);
        double sn, cs;
        sincos(ang, &sn, &cs);
        r[2 * k] = __dsub_rn(x[2 * k], __dmul_rn(rh, cs));
        r[2 * k + 1] = __dsub_rn(x[2 * k + 1], __dmul_rn(rh, sn));
        ss = __dadd_rn(ss, __dadd_rn(__dmul_rn(r[2 * k], r[2 * k]), __dmul_rn(r[2 * k + 1], r[2 * k + 1])));
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
      uint16_t rnb = f64_to_f16_bits(__dsqrt_rn(ss));
      if ((rnb & 0x7c00u) == 0x7c00u && lane == 0) atomicOr(a.status, kStatusRange);
#pragma unroll
      for (int i = 0; i < E; ++i) rbuf[lane * E + i] = r[i];
      __syncwarp();
      uint8_t* rec_bits = blk + L.off_ks + row * L.sg_bytes;
      for (int k = 0; k < (m + 31) / 32; ++k) {
        const int i = lane + 32 * k;
        double acc = 0.0;
        if (i < m) {
          const float* col = a.St + i;
#pragma unroll 8
          for (int jj = 0; jj < D; ++jj) acc = fma((double)__ldg(col + (size_t)jj * m), rbuf[jj], acc);
        }
        const unsigned word = __ballot_sync(kFull, i < m && acc >= 0.0);
        if (lane < 4 && 4 * k + lane < L.sg_bytes) rec_bits[4 * k + lane] = (uint8_t)(word >> (8 * lane));
      }
      if (lane == 0) reinterpret_cast<uint16_t*>(blk + L.off_krn)[row] = rnb;
    }

    // ---- pack code words LSB-first into the record ---------------------
    __syncwarp();
    const int nwords = L.kc_bytes / 4;
    for (int w = lane; w < nwords; w += 32) {
      const int bit0 = 32 * w;
      uint32_t word = 0;
      const int j0 = bit0 / bw, j1 = (bit0 + 31) / bw;
      for (int jj = j0; jj <= j1 && jj < D / 2; ++jj) {
        const int pos = jj * bw - bit0;
        const uint32_t c = cbuf[jj];
        word |= pos >= 0 ? (c << pos) : (c >> (-pos));
      }
      reinterpret_cast<uint32_t*>(rec_codes)[w] = word;
    }
    if (lane == 0) *rec_scale = s16b;
    __syncwarp();
  }
}

__global__ void ring_write_kernel(__half* ring_k, __half* ring_v, const __half* k_new,
                                  const __half* v_new, int units, int W, int d, int n,
                                  int first, int ring_pos) {
  const int chunks = d / 8;   // 16-byte chunks per token
  const int64_t per_unit = (int64_t)(n - first) * chunks;
  const int64_t total = 2 * (int64_t)units * per_unit;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const bool is_k = idx < total / 2;
    const int64_t j = is_k ? idx : idx - total / 2;
    const int unit = (int)(j / per_unit);
    const int64_t r = j % per_unit;
    const int i = first + (int)(r / chunks);
    const int c = (int)(r % chunks);
    const int slot = (int)(((int64_t)ring_pos + i) % W);
    const uint4* s = reinterpret_cast<const uint4*>((is_k ? k_new : v_new) + ((int64_t)unit * n + i) * d) + c;
    uint4* dst = reinterpret_cast<uint4*>((is_k ? ring_k : ring_v) + ((int64_t)unit * W + slot) * d) + c;
    *dst = *s;
  }
}

template <int D>
cudaError_t launch_encode_d(const EncodeArgs& a, cudaStream_t s) {
  const int warps = 8;
  const int64_t jobs = 2 * (int64_t)a.units * ((int64_t)a.nA + a.nB);
  if (jobs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (jobs + warps - 1) / warps;
  const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
  const size_t smem = (size_t)warps * D * sizeof(double) + (size_t)warps * (D / 2);
  encode_kernel<D><<<grid, warps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
  switch (a.L.d) {
    case 64: return launch_encode_d<64>(a, s);
    case 128: return launch_encode_d<128>(a, s);
    case 256: return launch_encode_d<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_ring_write(__half* ring_k, __half* ring_v, const __half* k_new,
                              const __half* v_new, int units, int W, int d, int n, int first,
                              int ring_pos, cudaStream_t s) {
  const int64_t total = 2 * (int64_t)units * (n - first) * (d / 8);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int grid = (int)(want < 4096 ? want : 4096);
  ring_write_kernel<<<grid, threads, 0, s>>>(ring_k, ring_v, k_new, v_new, units, W, d, n, first,
                                             ring_pos);
  return cudaGetLastError();
}

}  // namespace tq
