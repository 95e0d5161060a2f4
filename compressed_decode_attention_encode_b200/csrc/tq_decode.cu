// Decode attention straight from the packed cold cache plus the fp16 hot
// ring ("TurboQuant: optimización de memoria para KV caches en inferencia
// de LLMs", flow step 6: attention logits from the compressed cache;
// "Monarch v3 ...", "Bucle de Decodificación Simplificado": aggregate the hot
// and cold scores, softmax, apply).
//
// Three launches per call:
//   qprep    q' = R q (fp32 Hadamard butterflies), q'' = S q', both stored
//            as fp16 with a power-of-two scale per head.
//   attend   one CTA per (row, kv head, split).  A split streams either
//            64-token cold blocks or 64-token hot tiles through shared
//            memory.  Per warp and 16-token tile the three products run on
//            tensor cores (mma.sync m16n8k16, fp16 in, fp32 accumulate):
//              cold logits  [16 tok x d] . q'   -- A operand = LUT-dequantized
//                           polar pairs, one 32-bit LUT load per pair
//              QJL term     [16 tok x m] . q''  -- A operand = +-1 built from
//                           the sign bits with one shift and one LOP3
//              P V          [d x 16 tok] . P    -- P transposed in registers
//                           with movmatrix
//            with an online softmax across tiles (exp2 domain).  The GQA
//            group (G <= 8 query heads) is the n = 8 side of every MMA.
//   combine  merges the split partials, applies R^T once to the cold sum
//            (Hadamard butterflies), normalizes.
#include <cfloat>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 128;          // 4 warps; each takes 16 tokens of a 64-token block
constexpr float kNegInf = -INFINITY;
constexpr float kSqrtHalfPi = 1.2533141373155001f;   // sqrt(pi / 2)

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// +-1 fp16 pair from the two sign bits at positions 15 and 31 of (x << u):
// bit 1 -> +1.0 (0x3C00), bit 0 -> -1.0 (0xBC00).
__device__ __forceinline__ uint32_t sign_pair(uint32_t x, int u) {
  return ((x << u) & 0x80008000u) ^ 0xBC00BC00u;
}

// Loads NW 32-bit words of a bit stream starting at bit `start` of `rec`
// (4-byte aligned), re-based so that bit `start` becomes bit 0 of out[0].
template <int NW>
__device__ __forceinline__ void load_chunk(const uint8_t* rec, int start, uint32_t (&out)[NW]) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(rec) + (start >> 5);
  const int sh = start & 31;
  uint32_t raw[NW + 1];
#pragma unroll
  for (int i = 0; i <= NW; ++i) raw[i] = p[i];
#pragma unroll
  for (int i = 0; i < NW; ++i) out[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
}

// The BW-bit field at bit `pos` (a compile-time constant after unrolling).
template <int BW, int NW>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[NW], int pos) {
  const int wi = pos >> 5, bi = pos & 31;
  uint32_t v;
  if (bi + BW <= 32 || wi + 1 >= NW)
    v = w[wi] >> bi;
  else
    v = __funnelshift_r(w[wi], w[wi + 1], bi);
  return v & ((1u << BW) - 1u);
}

// Online-softmax step over one 16-token tile for the thread's two heads
// (2*tig, 2*tig+1).  l2[0..1]: token gid, l2[2..3]: token gid+8.  Returns the
// factor by which previously accumulated sums must be rescaled.
__device__ __forceinline__ void softmax_tile(const float (&l2)[4], float (&m_run)[2],
                                             float (&p)[4], float (&corr)[2]) {
  float t0 = fmaxf(l2[0], l2[2]), t1 = fmaxf(l2[1], l2[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    t0 = fmaxf(t0, __shfl_xor_sync(kFull, t0, o));
    t1 = fmaxf(t1, __shfl_xor_sync(kFull, t1, o));
  }
  const float n0 = fmaxf(m_run[0], t0), n1 = fmaxf(m_run[1], t1);
  const float r0 = n0 == kNegInf ? 0.f : n0, r1 = n1 == kNegInf ? 0.f : n1;
  corr[0] = exp2f(m_run[0] - r0);
  corr[1] = exp2f(m_run[1] - r1);
  p[0] = exp2f(l2[0] - r0);
  p[1] = exp2f(l2[1] - r1);
  p[2] = exp2f(l2[2] - r0);
  p[3] = exp2f(l2[3] - r1);
  m_run[0] = n0;
  m_run[1] = n1;
}

// ---------------------------------------------------------------------------
// q-prep
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) qprep_kernel(const QPrepArgs a) {
  __shared__ float sv[256];
  __shared__ float sq[256];
  __shared__ float red[32];
  const int h = blockIdx.x, t = threadIdx.x, D = a.d, M = a.m;
  for (int i = t; i < D; i += blockDim.x)
    sv[i] = __half2float(a.q[(size_t)h * D + i]) * (float)a.signs[i];
  __syncthreads();
  for (int hh = 1; hh < D; hh <<= 1) {
    for (int i = t; i < D; i += blockDim.x) {
      if (!(i & hh)) {
        const float x = sv[i], y = sv[i + hh];
        sv[i] = x + y;
        sv[i + hh] = x - y;
      }
    }
    __syncthreads();
  }
  const float inv = rsqrtf((float)D);
  float amax = 0.f;
  for (int i = t; i < D; i += blockDim.x) {
    sv[i] *= inv;
    amax = fmaxf(amax, fabsf(sv[i]));
  }
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  amax = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  const float al1 = amax > 0.f ? exp2f(-floorf(log2f(amax))) : 1.f;
  for (int i = t; i < D; i += blockDim.x) a.qrot[(size_t)h * D + i] = __float2half_rn(sv[i] * al1);
  __syncthreads();
  float bmax = 0.f;
  for (int i = t; i < M; i += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < D; ++j) acc = fmaf(__ldg(a.St + (size_t)j * M + i), sv[j], acc);
    sq[i] = acc;
    bmax = fmaxf(bmax, fabsf(acc));
  }
  for (int o = 16; o; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
  if ((t & 31) == 0) red[8 + (t >> 5)] = bmax;
  __syncthreads();
  bmax = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) bmax = fmaxf(bmax, red[8 + w]);
  const float al2 = bmax > 0.f ? exp2f(-floorf(log2f(bmax))) : 1.f;
  // sign-fragment order: for chunk tig (m/4 signs) and slot u < m/8 the pair
  // (q''[c + m/8 - 1 - u], q''[c + m/4 - 1 - u]), c = tig * m/4.
  const int Q4 = M / 4, H = M / 8;
  for (int i = t; i < M; i += blockDim.x) {
    const int tg = i / Q4, j = i % Q4;
    const int u = j < H ? (H - 1 - j) : (2 * H - 1 - j);
    const int pos = (tg * H + u) * 2 + (j < H ? 0 : 1);
    a.qsk[(size_t)h * M + pos] = __float2half_rn(sq[i] * al2);
  }
  if (t == 0) {
    a.qscale[2 * h] = 1.f / al1;
    a.qscale[2 * h + 1] = 1.f / al2;
  }
}

// ---------------------------------------------------------------------------
// attend
// ---------------------------------------------------------------------------
template <int D, int M, int BW>
struct AttendShape {
  static constexpr int P = D / 2;
  static constexpr int NT = D / 16;                 // k-steps of the K logits == PV m-tiles
  static constexpr int QS = M / 16;                 // k-steps of the QJL product
  static constexpr int KC = P * BW / 8;             // code bytes per vector
  static constexpr int SG = M / 8;                  // sign bytes per key
  static constexpr int TB = kTokensPerBlock;
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_KS = OFF_KC + TB * KC;
  static constexpr int OFF_KSC = OFF_KS + TB * SG;
  static constexpr int OFF_KRN = OFF_KSC + TB * 2;
  static constexpr int OFF_VC = OFF_KRN + TB * 2;
  static constexpr int OFF_VSC = OFF_VC + TB * KC;
  static constexpr int BLOCK = OFF_VSC + TB * 2;
  static constexpr int KBITS = (P / 4) * BW;        // bits of a thread's K chunk
  static constexpr int KW = (KBITS + 31) / 32;
  static constexpr int VBITS = (P / 8) * BW;        // bits of a thread's V chunk
  static constexpr int VW = (VBITS + 31) / 32;
  static constexpr int NLUT = 1 << BW;
  static constexpr int LUT_BYTES = NLUT * 32 * 4;   // one copy per lane: no bank conflicts
  static constexpr int RS = 2 * D + 16;             // padded hot row stride (bytes)
  static constexpr int HOT_BYTES = 2 * TB * RS;
  static constexpr int MERGE_BYTES = (64 + 4 * 8 * D) * 4;
  static constexpr int STAGE = (BLOCK > HOT_BYTES ? (BLOCK > MERGE_BYTES ? BLOCK : MERGE_BYTES)
                                                   : (HOT_BYTES > MERGE_BYTES ? HOT_BYTES : MERGE_BYTES));
  static constexpr int SMEM = LUT_BYTES + STAGE;
};

template <int D, int M, int BW>
__global__ void __launch_bounds__(kThreads) attend_kernel(const AttendArgs a) {
  using S = AttendShape<D, M, BW>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  uint8_t* stage = smem + S::LUT_BYTES;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int per_unit = a.ns_cold + a.ns_hot;
  const int unit = blockIdx.x / per_unit;
  const int split = blockIdx.x % per_unit;
  const bool hot = split >= a.ns_cold;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int G = a.G;
  const int head0 = b * a.Hq + kvh * G;
  const int Lr = (1 << a.L.b_r) - 1;
  const int tb = warp * 16;            // this warp's tokens inside a block / tile

  float m_run[2] = {kNegInf, kNegInf};
  float l_run[2] = {0.f, 0.f};
  float mp_run[2] = {kNegInf, kNegInf};
  float O[S::NT][4];
#pragma unroll
  for (int i = 0; i < S::NT; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;

  if (!hot) {
    // LUT of 'unit' pair reconstructions c_r * (cos, sin)(2 pi c_th / 2^b_th)
    const int bt = a.L.b_theta;
    for (int i = tid; i < S::NLUT * 32; i += kThreads) {
      const int w = i >> 5;
      const int cr = w >> bt, ct = w & ((1 << bt) - 1);
      float sn, cs;
      sincospif(2.0f * (float)ct / (float)(1 << bt), &sn, &cs);
      lut[i] = pack_h2((float)cr * cs, (float)cr * sn);
    }
    // B fragments: q' pairs (P/4)*tig + {2s, 2s+1}; q'' sign slots 2s, 2s+1
    uint32_t qf[S::NT][2], qs[S::QS][2];
    float kpol[2], kqjl[2];
    if (gid < G) {
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.qrot + (size_t)(head0 + gid) * D) + (S::P / 4) * tig;
      const uint32_t* qk = reinterpret_cast<const uint32_t*>(a.qsk + (size_t)(head0 + gid) * M) + tig * (M / 8);
#pragma unroll
      for (int s = 0; s < S::NT; ++s) { qf[s][0] = qp[2 * s]; qf[s][1] = qp[2 * s + 1]; }
#pragma unroll
      for (int s = 0; s < S::QS; ++s) { qs[s][0] = qk[2 * s]; qs[s][1] = qk[2 * s + 1]; }
    } else {
#pragma unroll
      for (int s = 0; s < S::NT; ++s) qf[s][0] = qf[s][1] = 0u;
#pragma unroll
      for (int s = 0; s < S::QS; ++s) qs[s][0] = qs[s][1] = 0u;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int g = 2 * tig + hh;
      kpol[hh] = g < G ? a.log2e_sigma * a.qscale[2 * (head0 + g)] / (float)Lr : 0.f;
      kqjl[hh] = g < G ? a.log2e_sigma * kSqrtHalfPi / (float)M * a.qscale[2 * (head0 + g) + 1] : 0.f;
    }

    const int64_t nblk = (a.n_cold + S::TB - 1) / S::TB;
    const int64_t blk0 = (int64_t)split * a.blocks_per_split;
    const int64_t blk1 = blk0 + a.blocks_per_split < nblk ? blk0 + a.blocks_per_split : nblk;
    const uint8_t* ubase = a.cold + (size_t)unit * a.L.blocks_per_unit * S::BLOCK;
    for (int64_t blk = blk0; blk < blk1; ++blk) {
      __syncthreads();
      const uint4* src = reinterpret_cast<const uint4*>(ubase + (size_t)blk * S::BLOCK);
      uint4* dst = reinterpret_cast<uint4*>(stage);
      for (int i = tid; i < S::BLOCK / 16; i += kThreads) dst[i] = __ldg(src + i);
      __syncthreads();
      const int nvalid = (int)((a.n_cold - blk * S::TB) < S::TB ? (a.n_cold - blk * S::TB) : S::TB);
      if (tb >= nvalid) continue;

      const int t0 = tb + gid, t1 = tb + gid + 8;
      // ---- cold logits: polar part -------------------------------------
      uint32_t k0[S::KW], k1[S::KW];
      load_chunk<S::KW>(stage + S::OFF_KC + t0 * S::KC, tig * S::KBITS, k0);
      load_chunk<S::KW>(stage + S::OFF_KC + t1 * S::KC, tig * S::KBITS, k1);
      float cp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < S::NT; ++s) {
        const uint32_t a0 = lut[(field<BW>(k0, (2 * s) * BW) << 5) + lane];
        const uint32_t a1 = lut[(field<BW>(k1, (2 * s) * BW) << 5) + lane];
        const uint32_t a2 = lut[(field<BW>(k0, (2 * s + 1) * BW) << 5) + lane];
        const uint32_t a3 = lut[(field<BW>(k1, (2 * s + 1) * BW) << 5) + lane];
        mma16816(cp, a0, a1, a2, a3, qf[s][0], qf[s][1]);
      }
      // ---- cold logits: QJL part ---------------------------------------
      uint32_t x0, x1;
      if constexpr (M == 128) {
        x0 = *reinterpret_cast<const uint32_t*>(stage + S::OFF_KS + t0 * S::SG + 4 * tig);
        x1 = *reinterpret_cast<const uint32_t*>(stage + S::OFF_KS + t1 * S::SG + 4 * tig);
      } else {
        const uint32_t c0 = *reinterpret_cast<const uint16_t*>(stage + S::OFF_KS + t0 * S::SG + 2 * tig);
        const uint32_t c1 = *reinterpret_cast<const uint16_t*>(stage + S::OFF_KS + t1 * S::SG + 2 * tig);
        x0 = ((c0 & 0xffu) << 8) | ((c0 >> 8) << 24);
        x1 = ((c1 & 0xffu) << 8) | ((c1 >> 8) << 24);
      }
      float cq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < S::QS; ++s)
        mma16816(cq, sign_pair(x0, 2 * s), sign_pair(x1, 2 * s), sign_pair(x0, 2 * s + 1),
                 sign_pair(x1, 2 * s + 1), qs[s][0], qs[s][1]);

      const __half* ksc = reinterpret_cast<const __half*>(stage + S::OFF_KSC);
      const __half* krn = reinterpret_cast<const __half*>(stage + S::OFF_KRN);
      const __half* vsc = reinterpret_cast<const __half*>(stage + S::OFF_VSC);
      const bool v0 = t0 < nvalid, v1 = t1 < nvalid;
      const float sk0 = __half2float(ksc[t0]), sk1 = __half2float(ksc[t1]);
      const float rn0 = __half2float(krn[t0]), rn1 = __half2float(krn[t1]);
      float l2[4];
      l2[0] = v0 ? fmaf(rn0 * kqjl[0], cq[0], sk0 * kpol[0] * cp[0]) : kNegInf;
      l2[1] = v0 ? fmaf(rn0 * kqjl[1], cq[1], sk0 * kpol[1] * cp[1]) : kNegInf;
      l2[2] = v1 ? fmaf(rn1 * kqjl[0], cq[2], sk1 * kpol[0] * cp[2]) : kNegInf;
      l2[3] = v1 ? fmaf(rn1 * kqjl[1], cq[3], sk1 * kpol[1] * cp[3]) : kNegInf;
      float p[4], corr[2];
      softmax_tile(l2, m_run, p, corr);
      l_run[0] = l_run[0] * corr[0] + p[0] + p[2];
      l_run[1] = l_run[1] * corr[1] + p[1] + p[3];

      // ---- V weights p * s16_v, kept on their own running max -----------
      const float lv0 = v0 ? log2f(__half2float(vsc[t0])) : kNegInf;
      const float lv1 = v1 ? log2f(__half2float(vsc[t1])) : kNegInf;
      float xv[4] = {l2[0] + lv0, l2[1] + lv0, l2[2] + lv1, l2[3] + lv1};
      float pv[4], co[2];
      softmax_tile(xv, mp_run, pv, co);
#pragma unroll
      for (int i = 0; i < S::NT; ++i) {
        O[i][0] *= co[0]; O[i][1] *= co[1]; O[i][2] *= co[0]; O[i][3] *= co[1];
      }
      const uint32_t pb0 = movmatrix_trans(pack_h2(pv[0], pv[1]));
      const uint32_t pb1 = movmatrix_trans(pack_h2(pv[2], pv[3]));

      // ---- P V: V codes of pairs (P/8)*gid + i for tokens 2tig(+1)(+8) ---
      uint32_t w0[S::VW], w1[S::VW], w2[S::VW], w3[S::VW];
      const uint8_t* vc = stage + S::OFF_VC;
      load_chunk<S::VW>(vc + (tb + 2 * tig) * S::KC, gid * S::VBITS, w0);
      load_chunk<S::VW>(vc + (tb + 2 * tig + 1) * S::KC, gid * S::VBITS, w1);
      load_chunk<S::VW>(vc + (tb + 2 * tig + 8) * S::KC, gid * S::VBITS, w2);
      load_chunk<S::VW>(vc + (tb + 2 * tig + 9) * S::KC, gid * S::VBITS, w3);
#pragma unroll
      for (int i = 0; i < S::NT; ++i) {
        const uint32_t L0 = lut[(field<BW>(w0, i * BW) << 5) + lane];
        const uint32_t L1 = lut[(field<BW>(w1, i * BW) << 5) + lane];
        const uint32_t L2 = lut[(field<BW>(w2, i * BW) << 5) + lane];
        const uint32_t L3 = lut[(field<BW>(w3, i * BW) << 5) + lane];
        mma16816(O[i], __byte_perm(L0, L1, 0x5410), __byte_perm(L0, L1, 0x7632),
                 __byte_perm(L2, L3, 0x5410), __byte_perm(L2, L3, 0x7632), pb0, pb1);
      }
    }
  } else {
    // ---- hot tiles: fp16 K / V through padded shared memory --------------
    uint32_t qh[S::NT][2];
    if (gid < G) {
      const __half* qp = a.q + (size_t)(head0 + gid) * D;
#pragma unroll
      for (int s = 0; s < S::NT; ++s) {
        qh[s][0] = *reinterpret_cast<const uint32_t*>(qp + 16 * s + 2 * tig);
        qh[s][1] = *reinterpret_cast<const uint32_t*>(qp + 16 * s + 8 + 2 * tig);
      }
    } else {
#pragma unroll
      for (int s = 0; s < S::NT; ++s) qh[s][0] = qh[s][1] = 0u;
    }
    const int ntiles = (a.n_hot + S::TB - 1) / S::TB;
    const int hs = split - a.ns_cold;
    const int tile0 = hs * a.tiles_per_split;
    const int tile1 = tile0 + a.tiles_per_split < ntiles ? tile0 + a.tiles_per_split : ntiles;
    constexpr int CH = D / 8;        // 16-byte chunks per token row
    for (int tile = tile0; tile < tile1; ++tile) {
      __syncthreads();
      for (int i = tid; i < 2 * S::TB * CH; i += kThreads) {
        const int kv = i / (S::TB * CH);
        const int rem = i % (S::TB * CH);
        const int r = rem / CH, c = rem % CH;
        const int slot = tile * S::TB + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (slot < a.n_hot)
          v = __ldg(reinterpret_cast<const uint4*>((kv ? a.hot_v : a.hot_k) + ((size_t)unit * a.W + slot) * D) + c);
        *reinterpret_cast<uint4*>(stage + kv * S::TB * S::RS + r * S::RS + c * 16) = v;
      }
      __syncthreads();
      const int nvalid = a.n_hot - tile * S::TB < S::TB ? a.n_hot - tile * S::TB : S::TB;
      if (tb >= nvalid) continue;
      const uint32_t kbase = smem_addr(stage);
      const uint32_t vbase = kbase + S::TB * S::RS;
      const int mi = lane >> 3, rr = lane & 7;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < S::NT; ++s) {
        uint32_t af[4];
        ldsm_x4(af, kbase + (tb + rr + (mi & 1) * 8) * S::RS + (16 * s + (mi >> 1) * 8) * 2);
        mma16816(c, af[0], af[1], af[2], af[3], qh[s][0], qh[s][1]);
      }
      const bool v0 = tb + gid < nvalid, v1 = tb + gid + 8 < nvalid;
      float l2[4];
      l2[0] = v0 ? a.log2e_sigma * c[0] : kNegInf;
      l2[1] = v0 ? a.log2e_sigma * c[1] : kNegInf;
      l2[2] = v1 ? a.log2e_sigma * c[2] : kNegInf;
      l2[3] = v1 ? a.log2e_sigma * c[3] : kNegInf;
      float p[4], corr[2];
      softmax_tile(l2, m_run, p, corr);
      l_run[0] = l_run[0] * corr[0] + p[0] + p[2];
      l_run[1] = l_run[1] * corr[1] + p[1] + p[3];
#pragma unroll
      for (int i = 0; i < S::NT; ++i) {
        O[i][0] *= corr[0]; O[i][1] *= corr[1]; O[i][2] *= corr[0]; O[i][3] *= corr[1];
      }
      const uint32_t pb0 = movmatrix_trans(pack_h2(p[0], p[1]));
      const uint32_t pb1 = movmatrix_trans(pack_h2(p[2], p[3]));
#pragma unroll
      for (int i = 0; i < S::NT; ++i) {
        uint32_t af[4];
        ldsm_x4_trans(af, vbase + (tb + rr + (mi >> 1) * 8) * S::RS + (16 * i + (mi & 1) * 8) * 2);
        mma16816(O[i], af[0], af[1], af[2], af[3], pb0, pb1);
      }
    }
    mp_run[0] = m_run[0];
    mp_run[1] = m_run[1];
  }

  // ---- finalize: per-warp state -> shared -> one partial per head -------
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l_run[0] += __shfl_xor_sync(kFull, l_run[0], o);
    l_run[1] += __shfl_xor_sync(kFull, l_run[1], o);
  }
  float f[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if (m_run[hh] == kNegInf) f[hh] = 0.f;
    else if (hot) f[hh] = 1.f;
    else f[hh] = exp2f(mp_run[hh] - m_run[hh]) / (float)Lr;
  }
  __syncthreads();
  float* mw = reinterpret_cast<float*>(stage);     // [4 warps][8 heads]
  float* lw = mw + 32;
  float* ow = mw + 64;                              // [4][8][D]
  if (gid == 0) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      mw[warp * 8 + 2 * tig + hh] = m_run[hh];
      lw[warp * 8 + 2 * tig + hh] = l_run[hh];
    }
  }
#pragma unroll
  for (int i = 0; i < S::NT; ++i) {
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2) {
      const int dim = hot ? (16 * i + gid + 8 * r2) : (2 * ((S::P / 8) * gid + i) + r2);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int g = 2 * tig + hh;
        ow[(warp * 8 + g) * D + dim] = O[i][2 * r2 + hh] * f[hh];
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int g = idx / D, dim = idx % D;
    float mx = kNegInf;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, mw[w * 8 + g]);
    float o = 0.f, l = 0.f;
    if (mx != kNegInf) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mv = mw[w * 8 + g];
        if (mv == kNegInf) continue;
        const float sc = exp2f(mv - mx);
        o += sc * ow[(w * 8 + g) * D + dim];
        l += sc * lw[w * 8 + g];
      }
    }
    float* pp = a.part + (((size_t)unit * a.max_splits + split) * G + g) * (D + 2);
    pp[2 + dim] = o;
    if (dim == 0) {
      pp[0] = mx;
      pp[1] = l;
    }
  }
}

// ---------------------------------------------------------------------------
// combine
// ---------------------------------------------------------------------------
__global__ void combine_kernel(const CombineArgs a) {
  __shared__ float buf[256];
  const int hg = blockIdx.x;
  const int b = hg / a.Hq, hq = hg % a.Hq;
  const int kvh = hq / a.G, g = hq % a.G;
  const int unit = b * a.Hkv + kvh;
  const int D = a.d, t = threadIdx.x;
  const int ns = a.ns_cold + a.ns_hot;
  const float* base = a.part + (size_t)unit * a.max_splits * a.G * (D + 2);
  float mx = kNegInf;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, base[((size_t)s * a.G + g) * (D + 2)]);
  float lsum = 0.f, oc = 0.f, oh = 0.f;
  if (mx != kNegInf) {
    for (int s = 0; s < ns; ++s) {
      const float* pp = base + ((size_t)s * a.G + g) * (D + 2);
      if (pp[0] == kNegInf) continue;
      const float w = exp2f(pp[0] - mx);
      lsum += w * pp[1];
      const float v = w * pp[2 + t];
      if (s < a.ns_cold) oc += v; else oh += v;
    }
  }
  buf[t] = oc;
  __syncthreads();
  for (int h = 1; h < D; h <<= 1) {
    const float x = buf[t], y = buf[t ^ h];
    __syncthreads();
    buf[t] = (t & h) ? (y - x) : (x + y);
    __syncthreads();
  }
  const float res = mx == kNegInf ? 0.f
                                  : (oh + (float)a.signs[t] * buf[t] * rsqrtf((float)D)) / lsum;
  a.out[(size_t)hg * D + t] = res;
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
typedef void (*AttendFn)(const AttendArgs);

template <int D, int M, int BW>
AttendFn attend_fn(int* smem) {
  *smem = AttendShape<D, M, BW>::SMEM;
  return attend_kernel<D, M, BW>;
}

template <int D, int M>
AttendFn pick_bw(int bw, int* smem) {
  switch (bw) {
    case 2: return attend_fn<D, M, 2>(smem);
    case 3: return attend_fn<D, M, 3>(smem);
    case 4: return attend_fn<D, M, 4>(smem);
    case 5: return attend_fn<D, M, 5>(smem);
    case 6: return attend_fn<D, M, 6>(smem);
    case 7: return attend_fn<D, M, 7>(smem);
    case 8: return attend_fn<D, M, 8>(smem);
  }
  return nullptr;
}

AttendFn pick_attend(const Layout& L, int* smem) {
  if (L.d == 64 && L.m == 64) return pick_bw<64, 64>(L.bw, smem);
  if (L.d == 64 && L.m == 128) return pick_bw<64, 128>(L.bw, smem);
  if (L.d == 128 && L.m == 64) return pick_bw<128, 64>(L.bw, smem);
  if (L.d == 128 && L.m == 128) return pick_bw<128, 128>(L.bw, smem);
  return nullptr;
}

}  // namespace

int attend_ctas_per_sm(const Layout& L) {
  int smem = 0;
  AttendFn fn = pick_attend(L, &smem);
  if (!fn) return 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem) != cudaSuccess) return 0;
  return n;
}

cudaError_t launch_qprep(const QPrepArgs& a, cudaStream_t s) {
  qprep_kernel<<<a.heads, 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
  int smem = 0;
  AttendFn fn = pick_attend(a.L, &smem);
  if (!fn) return cudaErrorInvalidValue;
  const int grid = a.units * (a.ns_cold + a.ns_hot);
  fn<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  combine_kernel<<<a.batch * a.Hq, a.d, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
