// Vector inner-product search over TurboQuant codes ("Compresión del caché
// KV de los LLM a 3 bits: TurboQuant de Google Research", section
// "Aplicaciones más allá de los LLMs": the same compressed vectors rank a
// database for vector search / RAG).
//
//   vec_encode_kernel   float32 vectors -> codes, one warp per vector; the
//                       float64 decision path of the KV encoder.
//   vec_qprep_kernel    q' = R q, q'' = S q' written as the fp16 A operand of
//                       the search MMAs, in the fragments' column order.
//   search_kernel       per CTA (8 warps): 64 queries x a contiguous run of
//                       database vectors.  The database side is dequantized
//                       straight into mma.sync B fragments (one shared LUT
//                       load per polar pair, scaled by the vector's
//                       s16/(2^b_r-1); sign bits become +-rn16*sqrt(pi/2)/m
//                       with one LOP3), so each looked-up register feeds 4
//                       MMAs.  Each thread compares its accumulators with
//                       its queries' current k-th best and appends only
//                       better candidates to a per-query buffer, which a
//                       warp re-selects when it could overflow.
//   topk_merge_kernel   merges the per-split candidate lists.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "tq_encode_core.cuh"

namespace tq {
namespace {

using enc::encode_vector_any;
using enc::kFull;
constexpr int kQT = 64;                  // queries per CTA
constexpr int kListK = 16;               // best candidates kept per (query, split); k <= kListK
constexpr int kMaxSplits = 32;           // database splits per search (grid y)
constexpr float kNegInf = -INFINITY;

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// (score, index) order of the result: higher score first, then lower index.
__device__ __forceinline__ bool better(float s, int i, float t, int j) {
  return s > t || (s == t && i < j);
}

// ---------------------------------------------------------------------------
// encode
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) vec_encode_kernel(const VecEncodeArgs a) {
  constexpr int E = D / 32, PL = E / 2, P = D / 2;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = blockDim.x >> 5;
  extern __shared__ double vsmem[];
  double* rbuf = vsmem + warp * D;
  uint8_t* codes = reinterpret_cast<uint8_t*>(vsmem + warps * D) + warp * (P + 64);
  uint32_t* bits = reinterpret_cast<uint32_t*>(codes + P);      // 8 words
  uint16_t* sc = reinterpret_cast<uint16_t*>(codes + P + 32);   // s16, rn16
  for (int64_t v = (int64_t)blockIdx.x * warps + warp; v < a.count; v += (int64_t)gridDim.x * warps) {
    const float* src = a.x + v * a.dim;
    auto load = [&](int ln, double (&x)[E]) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const int j = ln * E + i;
        x[i] = j < a.dim ? (double)src[j] : 0.0;
      }
    };
    if (lane < 8) bits[lane] = 0u;
    __syncwarp();
    encode_vector_any<D>(a.L, a.signs, a.St, a.inv_sqrt_d, a.status, load, true, rbuf, codes, bits,
                         sc, sc + 1);
    const int64_t g = a.start + v;
    uint8_t* dst = a.codes + g * P;
#pragma unroll
    for (int k = 0; k < PL; ++k) dst[lane * PL + k] = codes[lane * PL + k];
    if (lane < 8) reinterpret_cast<uint32_t*>(a.signs_out + g * 32)[lane] = bits[lane];
    if (lane == 0) {
      a.s16_out[g] = sc[0];
      a.rn16_out[g] = sc[1];
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// query prep: one warp per query
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) vec_qprep_kernel(const VecQPrepArgs a) {
  constexpr int E = D / 32, P = D / 2, PT = P / 4;
  constexpr int KA = D + 256;
  __shared__ float sq[8][D];
  __shared__ float sqq[8][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = blockIdx.x * 8 + warp;
  if (q >= a.nq) return;
  float x[E];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int j = lane * E + i;
    x[i] = j < a.dim ? a.q[(size_t)q * a.dim + j] * (float)a.signs[j] : 0.f;
  }
#pragma unroll
  for (int hh = 1; hh < D; hh <<= 1) {
    if (hh < E) {
#pragma unroll
      for (int i = 0; i < E; ++i)
        if (!(i & hh)) {
          const float p = x[i], r = x[i + hh];
          x[i] = p + r;
          x[i + hh] = p - r;
        }
    } else {
      const int lm = hh / E;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float o = __shfl_xor_sync(kFull, x[i], lm);
        x[i] = (lane & lm) ? (o - x[i]) : (x[i] + o);
      }
    }
  }
  const float inv = rsqrtf((float)D);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    x[i] *= inv;
    sq[warp][lane * E + i] = x[i];
    amax = fmaxf(amax, fabsf(x[i]));
  }
  __syncwarp();
  for (int i = lane; i < 256; i += 32) {
    float acc = 0.f;
    if (i < a.m)
      for (int j = 0; j < D; ++j) acc = fmaf(__ldg(a.St + (size_t)j * a.m + i), sq[warp][j], acc);
    sqq[warp][i] = acc;
    amax = fmaxf(amax, fabsf(acc));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
  const float al = amax > 0.f ? exp2f(-floorf(log2f(amax))) : 1.f;
  __syncwarp();
  __half* row = a.A + (size_t)q * KA;
  // polar columns: k-step s, column w of 16: pair PT*tig + 2s + (w >= 8)
  for (int c = lane; c < D; c += 32) {
    const int s = c / 16, w = c % 16;
    const int tig = (w % 8) / 2, e = w % 2;
    const int pair = PT * tig + 2 * s + (w >= 8 ? 1 : 0);
    row[c] = __float2half_rn(sq[warp][2 * pair + e] * al);
  }
  // QJL columns: sign word 2 tig + s/8, half2 slot u = 2 (s % 8) + (w >= 8)
  for (int c = lane; c < 256; c += 32) {
    const int s = c / 16, w = c % 16;
    const int tig = (w % 8) / 2, e = w % 2, r = w >= 8 ? 1 : 0;
    const int word = 2 * tig + s / 8, u = 2 * (s % 8) + r;
    const int idx = 32 * word + (e ? 31 - u : 15 - u);
    row[D + c] = __float2half_rn(idx < a.m ? sqq[warp][idx] * al : 0.f);
  }
  if (lane == 0) a.qscale[q] = 1.f / al;
}

// ---------------------------------------------------------------------------
// search
// ---------------------------------------------------------------------------
// Per CTA: kQT = 64 queries (4 MMA m-tiles, A operand in shared memory)
// against a contiguous run of the database, kStepVec = 128 vectors per step
// (8 warps x 2 n-tiles of 8).  Scores never go to shared memory: each
// thread compares its accumulators with the query's current k-th best
// (`thr`) and appends only better candidates to the query's buffer; a warp
// re-selects a query's k best whenever its buffer could overflow in the
// next step.
template <int D>
struct SearchShape {
  static constexpr int P = D / 2;
  static constexpr int PT = P / 4;            // code bytes per lane per vector
  static constexpr int KS_POL = D / 16;       // polar k-steps
  static constexpr int KS_QJL = 16;           // QJL k-steps (256 sign slots)
  static constexpr int KA = D + 256;
  static constexpr int AS = KA + 8;           // padded A row (halves)
  static constexpr int WARPS = 8;
  static constexpr int NJ = 2;                // n-tiles per warp per step
  static constexpr int STEP = WARPS * NJ * 8; // vectors per step
  static constexpr int CAP = kListK + STEP + 32;   // candidate slots per query
  static constexpr int OFF_CAND = kQT * AS * 2;
  static constexpr int OFF_CNT = OFF_CAND + kQT * CAP * 8;
  static constexpr int OFF_THR = OFF_CNT + kQT * 4;
  static constexpr int SMEM = OFF_THR + kQT * 4;
};

// Warp: replaces query q's candidates (n of them, (score, index) pairs) by
// its best min(n, K), in order, and returns the new count; *thr becomes the
// K-th best score (-inf while fewer than K are known).
template <int CAP, int K>
__device__ int select_top(float2* cand, int n, float* thr) {
  constexpr int PER = (CAP + 31) / 32;
  const int lane = threadIdx.x & 31;
  float sv[PER];
  int iv[PER];
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const int e = r * 32 + lane;
    const float2 c = e < n ? cand[e] : make_float2(kNegInf, 0.f);
    sv[r] = c.x;
    iv[r] = e < n ? __float_as_int(c.y) : 0x7fffffff;
  }
  __syncwarp();
  const int keep = n < K ? n : K;
  for (int k = 0; k < keep; ++k) {
    // this lane's best, then the warp's (score desc, index asc)
    float bs = sv[0];
    int bi = iv[0], br = 0;
#pragma unroll
    for (int r = 1; r < PER; ++r)
      if (better(sv[r], iv[r], bs, bi)) { bs = sv[r]; bi = iv[r]; br = r; }
    float ws = bs;
    int wi = bi;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float os = __shfl_xor_sync(kFull, ws, o);
      const int oi = __shfl_xor_sync(kFull, wi, o);
      if (better(os, oi, ws, wi)) { ws = os; wi = oi; }
    }
    if (bs == ws && bi == wi) {          // the owner drops it from its registers
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (r == br) { sv[r] = kNegInf; iv[r] = 0x7fffffff; }
    }
    if (lane == 0) cand[k] = make_float2(ws, __int_as_float(wi));
  }
  __syncwarp();
  if (lane == 0) *thr = keep == K ? cand[K - 1].x : kNegInf;
  __syncwarp();
  return keep;
}

template <int D, int K>
__global__ void __launch_bounds__(256, 1) search_kernel(const SearchArgs a) {
  using S = SearchShape<D>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ __align__(16) uint32_t lut[256 * 32];
  __half* As = reinterpret_cast<__half*>(smem);
  float2* cand = reinterpret_cast<float2*>(smem + S::OFF_CAND);
  int* cnt = reinterpret_cast<int*>(smem + S::OFF_CNT);
  float* thr = reinterpret_cast<float*>(smem + S::OFF_THR);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int q0 = blockIdx.x * kQT;
  const int nq_tile = a.nq - q0 < kQT ? a.nq - q0 : kQT;
  const int64_t per = (a.n + gridDim.y - 1) / gridDim.y;
  const int64_t v_lo = (int64_t)blockIdx.y * per;
  const int64_t v_hi = v_lo + per < a.n ? v_lo + per : a.n;

  // LUT of c_r * (cos, sin)(2 pi c_th / 2^b_th), one copy per lane
  for (int e = tid; e < 256 * 32; e += blockDim.x) {
    const int w = e >> 5;
    const int cr = w >> a.b_theta, ct = w & ((1 << a.b_theta) - 1);
    float sn, cs;
    sincospif(2.0f * (float)ct / (float)(1 << a.b_theta), &sn, &cs);
    const __half2 h = __floats2half2_rn((float)cr * cs, (float)cr * sn);
    lut[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  // A tile: the CTA's queries (rows past nq are zero)
  for (int i = tid; i < kQT * (S::KA / 8); i += blockDim.x) {
    const int r = i / (S::KA / 8), cc = i % (S::KA / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < nq_tile) v = *reinterpret_cast<const uint4*>(a.A + (size_t)(q0 + r) * S::KA + cc * 8);
    *reinterpret_cast<uint4*>(As + r * S::AS + cc * 8) = v;
  }
  for (int q = tid; q < kQT; q += blockDim.x) {
    cnt[q] = 0;
    thr[q] = kNegInf;
  }
  __syncthreads();

  const uint32_t a_base = smem_addr(As);
  const int mi = lane >> 3, rr = lane & 7;
  const uint32_t lane4 = (uint32_t)lane * 4u;
  const char* lutb = reinterpret_cast<const char*>(lut);

  for (int64_t c0 = v_lo; c0 < v_hi; c0 += S::STEP) {
    // ---- B operand data for this warp's n-tiles (8 vectors each) --------
    uint32_t cw[S::NJ][S::PT / 4];
    uint32_t sg[S::NJ][2];
    uint32_t sa[S::NJ], sb[S::NJ];
#pragma unroll
    for (int j = 0; j < S::NJ; ++j) {
      const int64_t v = c0 + warp * (8 * S::NJ) + j * 8 + gid;
      if (v < v_hi) {
        const uint32_t* cp = reinterpret_cast<const uint32_t*>(a.codes + v * S::P + S::PT * tig);
#pragma unroll
        for (int k = 0; k < S::PT / 4; ++k) cw[j][k] = __ldg(cp + k);
        const uint2 s2 = __ldg(reinterpret_cast<const uint2*>(a.signs + v * 32 + 8 * tig));
        sg[j][0] = s2.x;
        sg[j][1] = s2.y;
        const float s16 = __half2float(__ushort_as_half(__ldg(a.s16 + v)));
        const float rn = __half2float(__ushort_as_half(__ldg(a.rn16 + v)));
        const __half ah = __float2half_rn(s16 * a.inv_levels);
        const __half bh = __float2half_rn(rn * a.qjl_const);
        const uint32_t au = __half_as_ushort(ah), bu = __half_as_ushort(bh);
        sa[j] = au | (au << 16);
        sb[j] = (bu | (bu << 16)) | 0x80008000u;
      } else {
#pragma unroll
        for (int k = 0; k < S::PT / 4; ++k) cw[j][k] = 0u;
        sg[j][0] = sg[j][1] = 0u;
        sa[j] = 0u;
        sb[j] = 0u;        // +-0: vectors past the run score 0 (not appended below)
      }
    }
    float acc[4][S::NJ][4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int j = 0; j < S::NJ; ++j) acc[m][j][0] = acc[m][j][1] = acc[m][j][2] = acc[m][j][3] = 0.f;

    // ---- polar part ----------------------------------------------------
#pragma unroll
    for (int s = 0; s < S::KS_POL; ++s) {
      uint32_t af[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        ldsm_x4(af[m], a_base + ((16 * m + rr + (mi & 1) * 8) * S::AS + 16 * s + (mi >> 1) * 8) * 2);
#pragma unroll
      for (int j = 0; j < S::NJ; ++j) {
        const uint32_t w = cw[j][(2 * s) / 4];
        const uint32_t c0b = (w >> (8 * ((2 * s) % 4))) & 0xffu;
        const uint32_t c1b = (w >> (8 * ((2 * s + 1) % 4))) & 0xffu;
        const uint32_t b0 = hmul2_u32(*reinterpret_cast<const uint32_t*>(lutb + (c0b * 128u + lane4)), sa[j]);
        const uint32_t b1 = hmul2_u32(*reinterpret_cast<const uint32_t*>(lutb + (c1b * 128u + lane4)), sa[j]);
#pragma unroll
        for (int m = 0; m < 4; ++m) mma16816(acc[m][j], af[m][0], af[m][1], af[m][2], af[m][3], b0, b1);
      }
    }
    // ---- QJL part: +-b from the sign bits -------------------------------
#pragma unroll
    for (int s = 0; s < S::KS_QJL; ++s) {
      uint32_t af[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        ldsm_x4(af[m], a_base + ((16 * m + rr + (mi & 1) * 8) * S::AS + D + 16 * s + (mi >> 1) * 8) * 2);
      const int u = 2 * (s % 8);
#pragma unroll
      for (int j = 0; j < S::NJ; ++j) {
        const uint32_t x = sg[j][s / 8];
        const uint32_t b0 = ((x << u) & 0x80008000u) ^ sb[j];
        const uint32_t b1 = ((x << (u + 1)) & 0x80008000u) ^ sb[j];
#pragma unroll
        for (int m = 0; m < 4; ++m) mma16816(acc[m][j], af[m][0], af[m][1], af[m][2], af[m][3], b0, b1);
      }
    }
    // ---- candidates: scores at least the query's current k-th best -------
#pragma unroll
    for (int m = 0; m < 4; ++m) {
#pragma unroll
      for (int r2 = 0; r2 < 2; ++r2) {
        const int q = 16 * m + gid + 8 * r2;
        if (q >= nq_tile) continue;
        const float t = thr[q];
#pragma unroll
        for (int j = 0; j < S::NJ; ++j) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int64_t v = c0 + warp * (8 * S::NJ) + j * 8 + 2 * tig + c;
            const float sc = acc[m][j][2 * r2 + c];
            if (v < v_hi && sc >= t) {
              const int pos = atomicAdd(&cnt[q], 1);
              cand[q * S::CAP + pos] = make_float2(sc, __int_as_float((int)v));
            }
          }
        }
      }
    }
    __syncthreads();
    // ---- re-select where the next step could overflow a buffer ----------
    for (int q = warp; q < nq_tile; q += S::WARPS) {
      const int n = cnt[q];
      if (n > S::CAP - S::STEP) cnt[q] = select_top<S::CAP, K>(cand + q * S::CAP, n, thr + q);
    }
    __syncthreads();
  }
  // ---- this CTA's list per query --------------------------------------------
  for (int q = warp; q < nq_tile; q += S::WARPS) {
    const int n = select_top<S::CAP, K>(cand + q * S::CAP, cnt[q], thr + q);
    const size_t base = ((size_t)(q0 + q) * gridDim.y + blockIdx.y) * K;
    for (int j = lane; j < K; j += 32) {
      const float2 c = j < n ? cand[q * S::CAP + j] : make_float2(kNegInf, __int_as_float(0x7fffffff));
      a.part_s[base + j] = c.x;
      a.part_i[base + j] = __float_as_int(c.y);
    }
  }
}

// One thread per query: the k best of its nsplit candidate lists.
template <int K>
__global__ void topk_merge_kernel(const MergeArgs a) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= a.nq) return;
  float ts[K];
  int ti[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    ts[j] = kNegInf;
    ti[j] = 0x7fffffff;
  }
  const int lists = a.nsplit;
  const size_t base = (size_t)q * lists * K;
  for (int e = 0; e < lists * K; ++e) {
    float sv = a.part_s[base + e];
    int iv = a.part_i[base + e];
    if (!better(sv, iv, ts[K - 1], ti[K - 1])) continue;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (better(sv, iv, ts[j], ti[j])) {
        const float t = ts[j];
        const int ii = ti[j];
        ts[j] = sv;
        ti[j] = iv;
        sv = t;
        iv = ii;
      }
    }
  }
  const float sc = a.qscale[q];
  for (int j = 0; j < a.k; ++j) {
    a.scores[(size_t)q * a.k + j] = ts[j] * sc;
    a.idx[(size_t)q * a.k + j] = ti[j];
  }
}

template <int D>
cudaError_t launch_vec_encode_d(const VecEncodeArgs& a, cudaStream_t s) {
  if (a.count == 0) return cudaSuccess;
  const int warps = 8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (a.count + warps - 1) / warps;
  const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
  const size_t smem = (size_t)warps * D * sizeof(double) + (size_t)warps * (D / 2 + 64);
  vec_encode_kernel<D><<<grid, warps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_search_d(const SearchArgs& a, cudaStream_t s) {
  using S = SearchShape<D>;
  if (cudaFuncSetAttribute(search_kernel<D, kListK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           S::SMEM) != cudaSuccess)
    return cudaErrorInvalidValue;
  dim3 grid((a.nq + kQT - 1) / kQT, a.nsplit);
  search_kernel<D, kListK><<<grid, 32 * S::WARPS, S::SMEM, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vec_encode(const VecEncodeArgs& a, cudaStream_t s) {
  switch (a.L.d) {
    case 64: return launch_vec_encode_d<64>(a, s);
    case 128: return launch_vec_encode_d<128>(a, s);
    case 256: return launch_vec_encode_d<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_vec_qprep(const VecQPrepArgs& a, cudaStream_t s) {
  const int grid = (a.nq + 7) / 8;
  switch (a.d) {
    case 64: vec_qprep_kernel<64><<<grid, 256, 0, s>>>(a); break;
    case 128: vec_qprep_kernel<128><<<grid, 256, 0, s>>>(a); break;
    case 256: vec_qprep_kernel<256><<<grid, 256, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_search(const SearchArgs& a, cudaStream_t s) {
  switch (a.d) {
    case 64: return launch_search_d<64>(a, s);
    case 128: return launch_search_d<128>(a, s);
    case 256: return launch_search_d<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk_merge(const MergeArgs& a, cudaStream_t s) {
  topk_merge_kernel<16><<<(a.nq + 127) / 128, 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace tq

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace tq {
namespace {

constexpr size_t kVAlign = 256;
size_t vround(size_t x) { return (x + kVAlign - 1) / kVAlign * kVAlign; }

int pad_dim(int d_in) {
  int d = 64;
  while (d < d_in) d *= 2;
  return d;
}

struct VecCodesLayout {
  size_t codes, signs, s16, rn16, total;
};

VecCodesLayout vec_codes_layout(int d, int64_t n) {
  VecCodesLayout l{};
  size_t off = 0;
  l.codes = off; off += vround((size_t)n * (d / 2));
  l.signs = off; off += vround((size_t)n * 32);
  l.s16 = off;   off += vround((size_t)n * 2);
  l.rn16 = off;  off += vround((size_t)n * 2);
  l.total = off;
  return l;
}

struct VecWsLayout {
  size_t status, signs, St, A, qscale, part_s, part_i, total;
};

VecWsLayout vec_ws_layout(int d, int m, int max_q) {
  VecWsLayout w{};
  size_t off = 0;
  w.status = off; off += kVAlign;
  w.signs = off;  off += vround(sizeof(double) * d);
  w.St = off;     off += vround(sizeof(float) * (size_t)d * m);
  w.A = off;      off += vround((size_t)2 * max_q * (d + 256));
  w.qscale = off; off += vround(sizeof(float) * max_q);
  w.part_s = off; off += vround(sizeof(float) * (size_t)max_q * kMaxSplits * kListK);
  w.part_i = off; off += vround(sizeof(int) * (size_t)max_q * kMaxSplits * kListK);
  w.total = off;
  return w;
}

tq_status check_vec(const tq_vec_config* c) {
  if (!c) return TQ_ERR_INVALID_ARG;
  if (c->dim < 1 || c->b_r < 1 || c->b_theta < 1 || c->qjl_bits < 8 || c->qjl_bits % 8)
    return TQ_ERR_INVALID_ARG;
  if (c->dim > 256 || c->qjl_bits > 256) return TQ_ERR_UNSUPPORTED;
  if (c->b_r + c->b_theta != 8) return TQ_ERR_UNSUPPORTED;
  return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

struct tq_vec_index {
  tq_vec_config cfg;
  int d;
  int64_t n;
  int max_q;
  Layout L;
  VecCodesLayout C;
  VecWsLayout W;
  uint8_t* ws;
  int device;
  int num_sms;
};

extern "C" {

tq_status tq_vec_bytes(const tq_vec_config* cfg, int64_t n, int32_t max_queries,
                       size_t* codes_bytes, size_t* workspace_bytes) {
  tq_status st = check_vec(cfg);
  if (st != TQ_OK) return st;
  if (n < 0 || max_queries < 1) return TQ_ERR_INVALID_ARG;
  const int d = pad_dim(cfg->dim);
  if (codes_bytes) *codes_bytes = vec_codes_layout(d, n).total;
  if (workspace_bytes) *workspace_bytes = vec_ws_layout(d, cfg->qjl_bits, max_queries).total;
  return TQ_OK;
}

tq_status tq_vec_create(const tq_vec_config* cfg, int64_t n, int32_t max_queries,
                        void* workspace_mem, cudaStream_t stream, tq_vec_index** out) {
  tq_status st = check_vec(cfg);
  if (st != TQ_OK) return st;
  if (!out || !workspace_mem || n < 1 || max_queries < 1 || ((uintptr_t)workspace_mem % kVAlign))
    return TQ_ERR_INVALID_ARG;
  if (n > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;   // indices are int32
  tq_vec_index* v = new (std::nothrow) tq_vec_index();
  if (!v) return TQ_ERR_INVALID_ARG;
  v->cfg = *cfg;
  v->d = pad_dim(cfg->dim);
  v->n = n;
  v->max_q = max_queries;
  v->L = layout_of(v->d, cfg->b_r, cfg->b_theta, cfg->qjl_bits, 0);
  v->C = vec_codes_layout(v->d, n);
  v->W = vec_ws_layout(v->d, cfg->qjl_bits, max_queries);
  v->ws = (uint8_t*)workspace_mem;
  if (cudaGetDevice(&v->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&v->num_sms, cudaDevAttrMultiProcessorCount, v->device) != cudaSuccess) {
    delete v;
    return TQ_ERR_CUDA;
  }
  const int d = v->d, m = cfg->qjl_bits;
  std::vector<double> signs(d);
  std::vector<float> S((size_t)m * d), St((size_t)m * d);
  int8_t* sg = new int8_t[d];
  tq_rotation_signs(cfg->seed, d, sg);
  for (int i = 0; i < d; ++i) signs[i] = sg[i];
  delete[] sg;
  tq_qjl_matrix(cfg->seed, m, d, S.data());
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) St[(size_t)j * m + i] = S[(size_t)i * d + j];
  cudaError_t e = cudaMemsetAsync(v->ws + v->W.status, 0, kVAlign, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(v->ws + v->W.signs, signs.data(), sizeof(double) * d, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(v->ws + v->W.St, St.data(), sizeof(float) * St.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    delete v;
    return TQ_ERR_CUDA;
  }
  *out = v;
  return TQ_OK;
}

tq_status tq_vec_destroy(tq_vec_index* index) {
  delete index;
  return TQ_OK;
}

tq_status tq_encode_vectors(tq_vec_index* v, const float* x, int64_t start, int64_t count,
                            void* codes, cudaStream_t stream) {
  if (!v || !codes || start < 0 || count < 0 || start + count > v->n) return TQ_ERR_INVALID_ARG;
  if (count == 0) return TQ_OK;
  if (!x) return TQ_ERR_INVALID_ARG;
  VecEncodeArgs a{};
  a.x = x;
  a.start = start;
  a.count = count;
  a.dim = v->cfg.dim;
  a.L = v->L;
  a.signs = (const double*)(v->ws + v->W.signs);
  a.St = (const float*)(v->ws + v->W.St);
  a.inv_sqrt_d = 1.0 / std::sqrt((double)v->d);
  a.status = (int*)(v->ws + v->W.status);
  uint8_t* base = (uint8_t*)codes;
  a.codes = base + v->C.codes;
  a.signs_out = base + v->C.signs;
  a.s16_out = (uint16_t*)(base + v->C.s16);
  a.rn16_out = (uint16_t*)(base + v->C.rn16);
  return launch_vec_encode(a, stream) == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_ip_search(tq_vec_index* v, const void* codes, const float* q, int32_t nq, int32_t k,
                       float* scores, int32_t* idx, cudaStream_t stream) {
  if (!v || !codes || !q || !scores || !idx || nq < 1 || nq > v->max_q || k < 1 || k > kListK)
    return TQ_ERR_INVALID_ARG;
  VecQPrepArgs qa{};
  qa.q = q;
  qa.nq = nq;
  qa.dim = v->cfg.dim;
  qa.d = v->d;
  qa.m = v->cfg.qjl_bits;
  qa.signs = (const double*)(v->ws + v->W.signs);
  qa.St = (const float*)(v->ws + v->W.St);
  qa.A = (__half*)(v->ws + v->W.A);
  qa.qscale = (float*)(v->ws + v->W.qscale);
  if (launch_vec_qprep(qa, stream) != cudaSuccess) return TQ_ERR_CUDA;
  // one wave: query tiles x database splits ~ the SM count
  const int qtiles = (nq + 63) / 64;
  int nsplit = std::max(1, v->num_sms / qtiles);
  nsplit = std::min(nsplit, kMaxSplits);
  nsplit = (int)std::min<int64_t>(nsplit, (v->n + 127) / 128);
  SearchArgs sa{};
  const uint8_t* base = (const uint8_t*)codes;
  sa.A = qa.A;
  sa.codes = base + v->C.codes;
  sa.signs = base + v->C.signs;
  sa.s16 = (const uint16_t*)(base + v->C.s16);
  sa.rn16 = (const uint16_t*)(base + v->C.rn16);
  sa.n = v->n;
  sa.nq = nq;
  sa.d = v->d;
  sa.b_theta = v->cfg.b_theta;
  sa.nsplit = nsplit;
  sa.inv_levels = 1.0f / (float)((1 << v->cfg.b_r) - 1);
  sa.qjl_const = (float)(std::sqrt(M_PI / 2.0) / v->cfg.qjl_bits);
  sa.part_s = (float*)(v->ws + v->W.part_s);
  sa.part_i = (int*)(v->ws + v->W.part_i);
  if (launch_search(sa, stream) != cudaSuccess) return TQ_ERR_CUDA;
  MergeArgs ma{};
  ma.part_s = sa.part_s;
  ma.part_i = sa.part_i;
  ma.qscale = qa.qscale;
  ma.nq = nq;
  ma.nsplit = nsplit;
  ma.k = k;
  ma.scores = scores;
  ma.idx = idx;
  return launch_topk_merge(ma, stream) == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_export_vectors(tq_vec_index* v, const void* codes, int64_t start, int64_t count,
                            uint8_t* codes_out, uint8_t* bits_out, uint16_t* s16_out,
                            uint16_t* rn16_out, cudaStream_t stream) {
  if (!v || !codes || start < 0 || count < 0 || start + count > v->n) return TQ_ERR_INVALID_ARG;
  if (count == 0) return TQ_OK;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  const uint8_t* base = (const uint8_t*)codes;
  const int P = v->d / 2, mb = v->cfg.qjl_bits / 8;
  cudaError_t e = cudaSuccess;
  // bw = 8: the canonical LSB-first stream is one byte per pair
  if (codes_out) e = cudaMemcpy(codes_out, base + v->C.codes + start * P, (size_t)count * P, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && bits_out) {
    std::vector<uint8_t> tmp((size_t)count * 32);
    e = cudaMemcpy(tmp.data(), base + v->C.signs + start * 32, tmp.size(), cudaMemcpyDeviceToHost);
    for (int64_t i = 0; e == cudaSuccess && i < count; ++i) std::memcpy(bits_out + i * mb, tmp.data() + i * 32, mb);
  }
  if (e == cudaSuccess && s16_out) e = cudaMemcpy(s16_out, base + v->C.s16 + start * 2, (size_t)count * 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && rn16_out) e = cudaMemcpy(rn16_out, base + v->C.rn16 + start * 2, (size_t)count * 2, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // extern "C"
