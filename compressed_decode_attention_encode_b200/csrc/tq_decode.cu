// Decode attention straight from the packed cold cache plus the fp16 hot
// ring ("TurboQuant: optimización de memoria para KV caches en inferencia
// de LLMs", flow step 6: attention logits from the compressed cache;
// "Monarch v3 ...", "Bucle de Decodificación Simplificado": aggregate the hot
// and cold scores, softmax, apply).
//
// Three launches per call:
//   qprep    q' = R q (fp32 Hadamard butterflies) split into fp16 hi + lo
//            parts, q'' = S q' in fp16; power-of-two scale per head.
//   attend   one wave of CTAs.  Cold CTAs take equal contiguous runs of the
//            flattened (unit, 64-token block) list and stream them through a
//            multi-stage shared-memory ring filled by cp.async.bulk copies
//            (mbarrier completion, bounded waits).  Per warp and 16-token
//            tile the products run on tensor cores (mma.sync m16n8k16, fp16
//            in, fp32 accumulate):
//              cold logits [16 tok x d] . (q'hi + q'lo) -- A = LUT-dequantized
//                          polar pairs, one 32-bit LUT load per pair
//              QJL term    [16 tok x m] . q''        -- A = +-1 from the sign
//                          bits (one shift + one LOP3 per pair)
//              P V         [d x 16 tok] . P          -- P transposed in
//                          registers with movmatrix
//            with an online softmax (exp2 domain).  The GQA group (G <= 8
//            query heads) is the n = 8 side of every MMA.  Hot CTAs stream
//            fp16 tiles through padded shared memory (ldmatrix).
//   combine  merges the partials of each (row, head), applies R^T once to
//            the cold sum (Hadamard butterflies) and normalizes.
// A gated call (tq_decode_attention_gated) runs the gate of tq_gate.cu
// between qprep and attend; its attention kernel streams the cold blocks of
// the listed units only, split again over the same CTAs, and combine leaves
// out the cold partials of the heads that skipped.
#include <cfloat>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 128;          // 4 warps; each takes 16 tokens of a 64-token block
constexpr int kAttendMinBlocks = 4;    // attention CTAs per SM the shapes are sized for
constexpr int kSmemPerSm = 233472;     // shared memory per SM (bytes)
// Shared-window address of a kernel's dynamic shared memory when it has no
// static shared variables: the first kilobyte of a CTA's window is reserved
// for the system.  The attention kernel checks it and reports a layout
// error rather than reading a misaligned table.
constexpr int kDynSmemBase = 1024;
constexpr float kNegInf = -INFINITY;
constexpr float kSqrtHalfPi = 1.2533141373155001f;   // sqrt(pi / 2)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // bounded mbarrier waits

// ---- PTX helpers -----------------------------------------------------------
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

// Shared-memory loads of ring stages by shared-window address, volatile so
// that they stay after the stage's wait.

__device__ __forceinline__ uint2 lds_ring64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lds_ring32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of an mbarrier, giving up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Global -> shared bulk copy completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// +-1 fp16 pair from sign bits 15-u and 31-u of x: bit 1 -> +1.0 (0x3C00),
// bit 0 -> -1.0 (0xBC00).  Written as one shift and one three-input logic
// op ((x << u) & 0x80008000) ^ 0xBC00BC00 in PTX, which the compiler keeps
// as two instructions (its own lowering of the C++ form took three).
__device__ __forceinline__ uint32_t sign_pair(uint32_t x, int u) {
  uint32_t r;
  asm("{\n .reg .b32 s;\n shl.b32 s, %1, %2;\n lop3.b32 %0, s, 0x80008000, 0xBC00BC00, 0x6A;\n}"
      : "=r"(r)
      : "r"(x), "r"(u));
  return r;
}

// Byte offset in a LUT whose entries are 2^SH bytes apart, of the entry
// named by the BW-bit field at bit `pos` of the lane's word stream (`pos`
// is a compile-time constant after unrolling), plus `lane_off` (the lane's
// copy inside the entry): one shift (a funnel shift for a field straddling
// two words) and one three-input logic op, written in PTX so that the
// compiler keeps it at two instructions.
template <int BW, int SH, int NW>
__device__ __forceinline__ uint32_t lut_offset(const uint32_t (&w)[NW], int pos, uint32_t lane_off) {
  constexpr uint32_t kMask = ((1u << BW) - 1u) << SH;
  const int wi = pos >> 5, bi = pos & 31;
  uint32_t t, r;
  if (bi + BW <= 32 || wi + 1 >= NW) {
    if (bi >= SH) asm("shr.b32 %0, %1, %2;" : "=r"(t) : "r"(w[wi]), "r"(bi - SH));
    else asm("shl.b32 %0, %1, %2;" : "=r"(t) : "r"(w[wi]), "r"(SH - bi));
  } else {
    asm("shf.r.wrap.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(w[wi]), "r"(w[wi + 1]), "r"(bi - SH));
  }
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(t), "n"(kMask), "r"(lane_off));   // (t & m) | l
  return r;
}

// ---------------------------------------------------------------------------
// q-prep: HB = 256 / M heads per block (2 for m = 128), so that the grid
// spreads over the SMs.  One warp per head rotates q (butterflies in
// registers and across lanes); then every thread computes one element of
// S q' from S^T staged in shared memory (asynchronous copies issued before
// the rotation).
// ---------------------------------------------------------------------------
template <int D, int M>
__device__ __forceinline__ void qprep_body(const QPrepArgs& a);

template <int D, int M>
__global__ void __launch_bounds__(256) qprep_kernel(const QPrepArgs a) {
  // a gated call's gate kernel (a programmatic dependent) may start now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  qprep_body<D, M>(a);
  // launched as a programmatic dependent of the previous kernel: finish
  // only after that kernel has (its writes visible to what follows q-prep)
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D, int M>
__device__ __forceinline__ void qprep_body(const QPrepArgs& a) {
  constexpr int E = D / 32;
  constexpr int HB = 256 / M;            // heads per block
  __shared__ float sq[HB][D];
  __shared__ float sqq[HB][M];
  extern __shared__ float4 sst4[];       // S^T [D][M]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  async_copy_g2s(sst4, a.St, D * M * 4);       // lands while the rotation runs
  const float* sst = reinterpret_cast<const float*>(sst4);
  const int h = blockIdx.x * HB + warp;          // head of this warp (warps < HB)
  if (warp < HB) {
    const bool live = h < a.heads;
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i)
      x[i] = live ? __half2float(a.q[(size_t)h * D + lane * E + i]) * (float)a.signs[lane * E + i] : 0.f;
#pragma unroll
    for (int hh = 1; hh < D; hh <<= 1) {
      if (hh < E) {
#pragma unroll
        for (int i = 0; i < E; ++i)
          if (!(i & hh)) {
            const float p = x[i], q = x[i + hh];
            x[i] = p + q;
            x[i + hh] = p - q;
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
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float al1 = amax > 0.f ? exp2f(-floorf(log2f(amax))) : 1.f;
    if (live) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float v = x[i] * al1;
        const __half hi = __float2half_rn(v);
        a.qrot[(size_t)h * 2 * D + lane * E + i] = hi;
        a.qrot[(size_t)h * 2 * D + D + lane * E + i] = __float2half_rn(v - __half2float(hi));
      }
      if (lane == 0) a.qscale[2 * h] = 1.f / al1;
    }
  }
  async_copy_wait();
  __syncthreads();
  {
    const int hb = threadIdx.x / M, i = threadIdx.x % M;
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < D; ++j) acc = fmaf(sst[j * M + i], sq[hb][j], acc);
    sqq[hb][i] = acc;
  }
  __syncthreads();
  if (warp >= HB || h >= a.heads) return;
  float bmax = 0.f;
  for (int i = lane; i < M; i += 32) bmax = fmaxf(bmax, fabsf(sqq[warp][i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
  const float al2 = bmax > 0.f ? exp2f(-floorf(log2f(bmax))) : 1.f;
  // sign-fragment order: for chunk tig (m/4 signs) and slot u < m/8 the pair
  // (q''[c + m/8 - 1 - u], q''[c + m/4 - 1 - u]), c = tig * m/4.
  constexpr int Q4 = M / 4, H = M / 8;
  for (int i = lane; i < M; i += 32) {
    const int tg = i / Q4, j = i % Q4;
    const int u = j < H ? (H - 1 - j) : (2 * H - 1 - j);
    const int pos = (tg * H + u) * 2 + (j < H ? 0 : 1);
    a.qsk[(size_t)h * M + pos] = __float2half_rn(sqq[warp][i] * al2);
  }
  if (lane == 0) a.qscale[2 * h + 1] = 1.f / al2;
}

// ---------------------------------------------------------------------------
// attend
// ---------------------------------------------------------------------------
template <int D, int M, int BW>
struct AttendShape {
  static constexpr int P = D / 2;
  static constexpr int NT = D / 16;                 // k-steps of the K logits == PV m-tiles
  static constexpr int QS = M / 16;                 // k-steps of the QJL product
  static constexpr int PT = P / 4;                  // K pairs per lane (per token)
  static constexpr int PV = P / 8;                  // V pairs per lane (per token)
  static constexpr int KWT = (2 * PT * BW + 31) / 32;
  static constexpr int SW = (2 * (M / 4) + 31) / 32;
  static constexpr int VWT = (4 * PV * BW + 31) / 32;
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_KS = OFF_KC + 128 * KWT;
  static constexpr int OFF_KSC = OFF_KS + 128 * SW;
  static constexpr int OFF_VC = OFF_KSC + 64;
  static constexpr int OFF_VSC = OFF_VC + 128 * VWT;
  static constexpr int TT = OFF_VSC + 32;           // tile bytes
  static constexpr int TB = kTokensPerBlock;
  static constexpr int BLOCK = kTilesPerBlock * TT;
  static constexpr int NLUT = 1 << BW;
  // Two LUTs of fp16 pairs, one 4-byte copy per lane per entry (entries
  // 128 bytes apart): hi (keys and values), then lo (the keys' rounding
  // remainder).  The hi table starts on a LUT_ALIGN boundary of the shared
  // window, so a lookup's address is (table | entry << 7 | lane << 2) -- one
  // logic op -- and the lo entry is the same address + LUT_BYTES.
  static constexpr int LUT_BYTES = NLUT * 32 * 4;
  static constexpr int LUT_ALIGN = 128 << BW;
  static constexpr int RS = 2 * D + 16;             // padded hot row stride (bytes)
  static constexpr int HOT_BYTES = TB * RS;          // one hot tile, K then V
  static constexpr int MERGE_BYTES = (64 + 8 * D) * 4;
  // up to 8 stages per warp: 4 x 8 barriers, the abort flag
  static constexpr int BAR_BYTES = 4 * 8 * 8 + 16;
  // Dynamic shared memory: [ring | pad | LUT hi | LUT lo | merge | barriers],
  // laid out for a dynamic base at shared address kDynSmemBase.
  static constexpr int ring_bytes(int ns) { return ns * BLOCK > HOT_BYTES ? ns * BLOCK : HOT_BYTES; }
  static constexpr int lut_off(int ns) {
    return (kDynSmemBase + ring_bytes(ns) + LUT_ALIGN - 1) / LUT_ALIGN * LUT_ALIGN - kDynSmemBase;
  }
  static constexpr int smem_bytes(int ns) { return lut_off(ns) + 2 * LUT_BYTES + MERGE_BYTES + BAR_BYTES; }
  // ring stages: as many as fit when kAttendMinBlocks CTAs share an SM (2 to 8)
  static constexpr int SMEM_PER_CTA = kSmemPerSm / kAttendMinBlocks - 1024;
  static constexpr int pick_ns() {
    int ns = 2;
    for (int k = 3; k <= 8; ++k)
      if (smem_bytes(k) <= SMEM_PER_CTA) ns = k;
    return ns;
  }
  static constexpr int NS = pick_ns();
  static constexpr int OFF_LUT = lut_off(NS);
  static constexpr int OFF_MERGE = OFF_LUT + 2 * LUT_BYTES;
  static constexpr int OFF_BAR = OFF_MERGE + MERGE_BYTES;
  static constexpr int SMEM = smem_bytes(NS);
};

// 2-word-major per-lane words of a tile plane (see Layout).
template <int NW>
__device__ __forceinline__ void load_lane_words(uint32_t plane, int lane, uint32_t (&w)[NW]) {
#pragma unroll
  for (int g = 0; 2 * g < NW; ++g) {
    if (2 * g + 1 < NW) {
      const uint2 v = lds_ring64(plane + g * 256 + lane * 8);
      w[2 * g] = v.x;
      w[2 * g + 1] = v.y;
    } else {
      w[2 * g] = lds_ring32(plane + g * 256 + lane * 4);
    }
  }
}

// Spreads two 16-bit sign chunks so that slot u's bits land at 15 and 31
// after a left shift by u (m = 64 layout).
__device__ __forceinline__ uint32_t spread16(uint32_t c) {
  return ((c & 0xffu) << 8) | ((c >> 8 & 0xffu) << 24);
}

constexpr float kPvMax = 256.f;        // V weights p * s16_v stay <= 2^8 (fp16 operands)
constexpr float kPMax = 0x1p100f;      // softmax numerators p stay <= 2^100 (fp32 sums)
constexpr float kPRange = 100.f;

// Per-warp softmax / accumulator state for one unit: the reference `ref`
// (log2 domain) of the numerators p = 2^(l - ref) summed in `l_run`, and
// the accumulators O of the V weights p * s16_v.  A lane holds HPL query
// heads: 2 (heads 2 tig, 2 tig + 1: an MMA column per head) or 1 (head
// tig: the packed layout, where columns 2 tig and 2 tig + 1 carry the same
// head and the O columns are duplicates).
template <int NT, int HPL>
struct WarpState {
  float ref[HPL], l_run[HPL];
  float O[NT][4];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int h = 0; h < HPL; ++h) {
      ref[h] = kNegInf;
      l_run[h] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;
  }
};

// Online softmax over one 16-token tile with a lazily moved reference.
// l2: log2-domain logits, entry j for token gid + 8 (j / HPL) and the
// lane's head j % HPL; sv0 / sv1: the two tokens' V weights (the V
// record's s16, or 1 for hot tokens).  Produces p = 2^(l2 - ref) (added to
// l_run) and pv = p * sv (the V weights).  The reference moves -- one warp
// reduction, and a rescale of the sums -- only when some pv would exceed
// 2^8 or some p 2^100, so every pv fits fp16.
template <int NT, int HPL>
__device__ __forceinline__ void softmax_step(WarpState<NT, HPL>& st, const float (&l2)[2 * HPL],
                                             float sv0, float sv1, float (&pv)[2 * HPL]) {
  constexpr int J = 2 * HPL;
  float p[J];
  bool ok = true;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    p[j] = fast_exp2(l2[j] - st.ref[j % HPL]);
    pv[j] = p[j] * (j < HPL ? sv0 : sv1);
    ok &= (pv[j] <= kPvMax) & (p[j] <= kPMax);   // false for NaN (no reference yet)
  }
  if (!__all_sync(kFull, ok)) {
    // new reference: max over the tile of max(l2 + log2 sv, l2 - 100)
    float t[HPL];
#pragma unroll
    for (int h = 0; h < HPL; ++h) t[h] = kNegInf;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const float tau = fmaxf(l2[j] + fast_log2(j < HPL ? sv0 : sv1), l2[j] - kPRange);
      t[j % HPL] = fmaxf(t[j % HPL], tau);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1)
#pragma unroll
      for (int h = 0; h < HPL; ++h) t[h] = fmaxf(t[h], __shfl_xor_sync(kFull, t[h], o));
    float corr[HPL];
#pragma unroll
    for (int h = 0; h < HPL; ++h) {
      const float nr = fmaxf(st.ref[h], t[h]);
      corr[h] = st.ref[h] == kNegInf ? 0.f : fast_exp2(st.ref[h] - nr);
      st.ref[h] = nr;
      st.l_run[h] *= corr[h];
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      st.O[i][0] *= corr[0]; st.O[i][1] *= corr[HPL - 1];
      st.O[i][2] *= corr[0]; st.O[i][3] *= corr[HPL - 1];
    }
#pragma unroll
    for (int j = 0; j < J; ++j) {
      p[j] = fast_exp2(l2[j] - st.ref[j % HPL]);
      pv[j] = p[j] * (j < HPL ? sv0 : sv1);
    }
  }
#pragma unroll
  for (int h = 0; h < HPL; ++h) st.l_run[h] += p[h] + p[HPL + h];
}

// The PV MMA's B fragments (P^T: tokens x head columns) from the V weights.
template <int HPL>
__device__ __forceinline__ void pv_fragments(const float (&pv)[2 * HPL], uint32_t& pb0, uint32_t& pb1) {
  if constexpr (HPL == 2) {
    pb0 = movmatrix_trans(pack_h2(pv[0], pv[1]));
    pb1 = movmatrix_trans(pack_h2(pv[2], pv[3]));
  } else {                     // the head's weight in both of its columns
    pb0 = movmatrix_trans(pack_h2(pv[0], pv[0]));
    pb1 = movmatrix_trans(pack_h2(pv[1], pv[1]));
  }
}

// Merges the 4 warps' states into one partial {m, l, o[D]} per head and
// writes it to `dst` ([G][D + 2]).  Lane (gid, tig) holds heads
// HPL * tig + hh (heads >= G are dropped).  Called by all threads of the
// CTA; uses the merge area: per-warp m / l, then per-warp o rows summed by
// the threads.
template <int D, int NT, int HPL>
__device__ __forceinline__ void flush_partial(WarpState<NT, HPL>& st, bool hot, float inv_levels, int G,
                                              float* merge, float* dst) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1)
#pragma unroll
    for (int h = 0; h < HPL; ++h) st.l_run[h] += __shfl_xor_sync(kFull, st.l_run[h], o);
  float* mw = merge;          // [4 warps][8 heads]
  float* lw = merge + 32;
  float* ow = merge + 64;     // [8 heads][D]
  if (gid == 0) {
#pragma unroll
    for (int hh = 0; hh < HPL; ++hh) {
      mw[warp * 8 + HPL * tig + hh] = st.ref[hh];
      lw[warp * 8 + HPL * tig + hh] = st.l_run[hh];
    }
  }
  for (int i = tid; i < 8 * D; i += kThreads) ow[i] = 0.f;
  __syncthreads();
  float f[HPL];
#pragma unroll
  for (int hh = 0; hh < HPL; ++hh) {
    const int g = HPL * tig + hh;
    float mx = kNegInf;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, mw[w * 8 + g]);
    f[hh] = st.ref[hh] == kNegInf ? 0.f : fast_exp2(st.ref[hh] - mx) * (hot ? 1.f : inv_levels);
  }
  constexpr int P8 = D / 16;   // (D/2) / 8 pairs per gid for the cold mapping
  // the 4 warps add their rows in turn: no two threads touch one word at once
  for (int w = 0; w < 4; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < NT; ++i) {
#pragma unroll
        for (int r2 = 0; r2 < 2; ++r2) {
          const int dim = hot ? (16 * i + gid + 8 * r2) : (2 * (P8 * gid + i) + r2);
#pragma unroll
          for (int hh = 0; hh < HPL; ++hh) {
            const int g = HPL * tig + hh;
            if (g < G && f[hh] != 0.f) ow[g * D + dim] += st.O[i][2 * r2 + hh] * f[hh];
          }
        }
      }
    }
    __syncthreads();
  }
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int g = idx / D, dim = idx % D;
    float* pp = dst + g * (D + 2);
    pp[2 + dim] = ow[g * D + dim];
    if (dim == 0) {
      float mx = kNegInf;
#pragma unroll
      for (int w = 0; w < 4; ++w) mx = fmaxf(mx, mw[w * 8 + g]);
      float l = 0.f;
      if (mx != kNegInf) {
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (mw[w * 8 + g] != kNegInf) l += fast_exp2(mw[w * 8 + g] - mx) * lw[w * 8 + g];
      }
      pp[0] = mx;
      pp[1] = l;
    }
  }
  __syncthreads();
}

// PACK (groups of at most 4 query heads): the MMA's 8 columns carry
// [q'_hi | q'_lo] of the 4 heads, so the K-logit products take 2 MMAs per
// k-step instead of 3; lanes tig and tig ^ 2 then hold the same two heads
// 2 * (tig & 1) + hh.  Without PACK (8 heads) lane (gid, tig) holds heads
// 2 * tig + hh.
template <int D, int M, int BW, bool PACK, bool GATE>
__global__ void __launch_bounds__(kThreads, kAttendMinBlocks) attend_kernel(const AttendArgs a) {
  using S = AttendShape<D, M, BW>;
  extern __shared__ __align__(128) uint8_t smem[];
  // Separate 4-byte hi and lo entries (rather than one 8-byte entry) let
  // each looked-up register land directly in the MMA's operand registers.
  uint32_t* lhi_w = reinterpret_cast<uint32_t*>(smem + S::OFF_LUT);
  uint32_t* llo_w = lhi_w + S::NLUT * 32;
  uint8_t* ring = smem;
  float* merge = reinterpret_cast<float*>(smem + S::OFF_MERGE);
  // Each warp streams its own tiles (tile `warp` of every block of the
  // CTA's run) through its own NS-stage ring: barriers [4][NS], and a
  // CTA-wide abort flag.
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::OFF_BAR + 8 * 4 * S::NS);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.G;
  const int Lr = (1 << a.L.b_r) - 1;
  const float inv_levels = 1.f / (float)Lr;
  const int tb = warp * 16;            // this warp's tokens inside a block / tile
  const uint32_t lut_sa = smem_addr(lhi_w);
  if (lut_sa & (S::LUT_ALIGN - 1)) {   // dynamic base not where the layout assumes
    if (tid == 0) atomicOr(a.status, kStatusLayout);
    return;
  }
  const uint32_t lane_lut = lut_sa | ((uint32_t)lane * 4u);   // this lane's copy, hi table
  auto lut_hi = [&](uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
  };
  auto lut_lo = [&](uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(S::LUT_BYTES));
    return v;
  };
  const SplitPlan& pl = a.plan;
  const int slots = pl.slots_cold + pl.slots_hot;
  constexpr int HPL = PACK ? 1 : 2;      // query heads per lane on the cold path
  WarpState<S::NT, HPL> st;
  st.reset();

  const int c = blockIdx.x;
  // Ungated: the cold runs cover every unit.  Gated: they cover the units
  // of the active list (position p reads unit alist[p]), split again over
  // at most the plan's cold CTAs.
  int64_t g_bpc = 0, g_units = 0;
  int g_ctas = 0;
  if constexpr (GATE) {
    g_units = *a.n_active;
    gated_cold_split(g_units, pl.cold_blocks, pl.cold_ctas, &g_bpc, &g_ctas);
  }
  // (ungated, these stay reads of the launch parameters: no registers held)
  auto cold_bpc = [&]() -> int64_t {
    if constexpr (GATE) return g_bpc; else return pl.cold_bpc;
  };
  auto cold_units = [&]() -> int64_t {
    if constexpr (GATE) return g_units; else return a.units;
  };
  if (c < (GATE ? g_ctas : pl.cold_ctas)) {
    // ============ cold run: blocks [c * bpc, (c + 1) * bpc) ============
    const int64_t nb = pl.cold_blocks;
    const int64_t total = cold_units() * nb;
    const int64_t f_lo = (int64_t)c * cold_bpc();
    const int64_t f_hi = f_lo + cold_bpc() < total ? f_lo + cold_bpc() : total;
    const int nblk = (int)(f_hi - f_lo);
    const int nbi = (int)nb;
    const uint32_t bar_w = smem_addr(bars) + 8 * S::NS * warp;           // this warp's barriers
    const uint32_t ring_w = smem_addr(ring) + S::NS * S::TT * warp;      // this warp's stages
    // The warp's tile stream: `nsrc` is the next tile to fetch (block
    // `nblk_b` of its unit); it advances a block at a time and skips a
    // unit's unused blocks at the unit's end.  `issued` counts the copies.
    const uint8_t* nsrc;
    int nblk_b = 0, issued = 0;
    int fpos = 0;                        // gated: active-list position of nsrc's unit
    const size_t unit_gap = (size_t)(a.L.blocks_per_unit - nb) * S::BLOCK;
    {
      const int64_t u = f_lo / nb;
      nblk_b = (int)(f_lo - u * nb);
      fpos = (int)u;
      const int64_t uid = GATE ? (int64_t)a.alist[u] : u;
      nsrc = a.cold + ((size_t)uid * a.L.blocks_per_unit + (size_t)nblk_b) * S::BLOCK + warp * S::TT;
    }
    auto fetch_next = [&](int s) {       // lane 0: the next tile into stage s
      mbar_expect_tx(bar_w + 8 * s, S::TT);
      bulk_g2s(ring_w + s * S::TT, nsrc, S::TT, bar_w + 8 * s);
      ++issued;
      nsrc += S::BLOCK;
      if (++nblk_b == nbi) {
        nblk_b = 0;
        if constexpr (GATE)   // alist[n_active] exists (and is 0) for the run's last step
          nsrc = a.cold + (size_t)a.alist[++fpos] * a.L.blocks_per_unit * S::BLOCK + warp * S::TT;
        else
          nsrc += unit_gap;
      }
    };
    if (tid == 0) *abort_flag = 0;
    if (lane == 0) {
      for (int s = 0; s < S::NS; ++s) mbar_init(bar_w + 8 * s, 1);
      fence_barrier_init();
      for (int s = 0; s < S::NS && s < nblk; ++s) fetch_next(s);
    }
    // LUTs of 'unit' pair reconstructions c_r * (cos, sin)(2 pi c_th / 2^b_th):
    // keys as fp16 hi + lo (the lo part removes the fp16 rounding of the
    // table from the logits), values as fp16.
    {
      // 2^bw distinct entries (float64 sincospi once each), then one copy
      // per lane; the merge area is free at this point.
      const int bt = a.L.b_theta;
      uint2* base = reinterpret_cast<uint2*>(merge);
      for (int e = tid; e < S::NLUT; e += kThreads) {
        const int cr = e >> bt, ct = e & ((1 << bt) - 1);
        double sn, cs;
        sincospi(2.0 * (double)ct / (double)(1 << bt), &sn, &cs);
        const float x = (float)((double)cr * cs), y = (float)((double)cr * sn);
        const __half hx = __float2half_rn(x), hy = __float2half_rn(y);
        base[e] = make_uint2(pack_h2(__half2float(hx), __half2float(hy)),
                               pack_h2(x - __half2float(hx), y - __half2float(hy)));
      }
      __syncthreads();
      for (int i = tid; i < S::NLUT * 32; i += kThreads) {
        const uint2 e = base[i >> 5];
        lhi_w[i] = e.x;
        llo_w[i] = e.y;
      }
    }
    __syncthreads();

    // B operands of the K-logit MMAs (per k-step) and of the QJL MMAs.
    //   PACK:  bq = q'_hi / q'_lo in the even / odd column of each head; both
    //          A_hi and A_lo multiply it (the odd column's A_lo q'_lo term is
    //          2^-22 of the logit, and makes the product exact)
    //   else:  bq = q'_hi, bq2 = q'_lo
    constexpr int kAccSplit = PACK ? 2 : 1;    // independent accumulator chains
    uint32_t bq[S::NT][2], bq2[PACK ? 1 : S::NT][2], qs[S::QS][2];
    float kpol[HPL], kqjl[HPL];
    int unit_cur = -1;                    // active-list position when gated
    int uid_cur = 0;                      // gated: the unit itself (alist[unit_cur])
    int slot_cur = 0;
    bool aborted = false;
    int unit = (int)(f_lo / nb);          // advanced incrementally: no division per block
    int blk = (int)(f_lo - (int64_t)unit * nb);   // block inside the unit (< 2^31)
    const int tail = (int)(a.n_cold - (int64_t)(nbi - 1) * S::TB);   // valid tokens of a unit's last block
    for (int i = 0; i < nblk; ++i, ++blk) {
      if (blk == nbi) {
        blk = 0;
        ++unit;
      }
      if (unit != unit_cur) {
        if (unit_cur >= 0) {
          flush_partial<D, S::NT, HPL>(st, false, inv_levels, G, merge,
                                  a.part + (((size_t)(GATE ? uid_cur : unit_cur) * slots + slot_cur) * G) * (D + 2));
          st.reset();
        }
        unit_cur = unit;
        if constexpr (GATE) uid_cur = a.alist[unit];
        slot_cur = c - (int)(((int64_t)unit * nb) / cold_bpc());
        const int uid = GATE ? uid_cur : unit;
        const int b = uid / a.Hkv, kvh = uid % a.Hkv;
        const int head0 = b * a.Hq + kvh * G;
        // B column gid: head gid (8 heads) or, packed, head gid / 2 with
        // column parity 0 = q'_hi, 1 = q'_lo (QJL and the A_lo product use
        // the even columns only)
        const int hcol = PACK ? (gid >> 1) : gid;
        const bool odd = PACK && (gid & 1);
        if (hcol < G) {
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.qrot + (size_t)(head0 + hcol) * 2 * D) + S::PT * tig;
          const uint32_t* qk = reinterpret_cast<const uint32_t*>(a.qsk + (size_t)(head0 + hcol) * M) + tig * (M / 8);
          const int o1 = odd ? S::P : 0;
#pragma unroll
          for (int s = 0; s < S::NT; ++s) {
            bq[s][0] = qp[o1 + 2 * s];
            bq[s][1] = qp[o1 + 2 * s + 1];
            if constexpr (!PACK) {
              bq2[s][0] = qp[S::P + 2 * s];
              bq2[s][1] = qp[S::P + 2 * s + 1];
            }
          }
#pragma unroll
          for (int s = 0; s < S::QS; ++s) {
            qs[s][0] = odd ? 0u : qk[2 * s];
            qs[s][1] = odd ? 0u : qk[2 * s + 1];
          }
        } else {
#pragma unroll
          for (int s = 0; s < S::NT; ++s) bq[s][0] = bq[s][1] = 0u;
          if constexpr (!PACK) {
#pragma unroll
            for (int s = 0; s < S::NT; ++s) bq2[s][0] = bq2[s][1] = 0u;
          }
#pragma unroll
          for (int s = 0; s < S::QS; ++s) qs[s][0] = qs[s][1] = 0u;
        }
#pragma unroll
        for (int hh = 0; hh < HPL; ++hh) {
          const int g = HPL * tig + hh;
          kpol[hh] = g < G ? a.log2e_sigma * a.qscale[2 * (head0 + g)] * inv_levels : 0.f;
          kqjl[hh] = g < G ? a.log2e_sigma * kSqrtHalfPi / (float)M * a.qscale[2 * (head0 + g) + 1] : 0.f;
        }
      }
      // ---- wait for this tile's stage of the warp's ring --------------------
      const int stage = i % S::NS;
      if (!aborted) {
        const bool got = mbar_wait_bounded(bar_w + 8 * stage, (uint32_t)((i / S::NS) & 1));
        if (!__all_sync(kFull, got)) {
          aborted = true;
          if (lane == 0) *abort_flag = 1;
        }
      }
      const int left = (blk == nbi - 1 ? tail : S::TB) - tb;
      if (!aborted && left > 0) {
      const int nvalid = left < 16 ? (int)left : 16;     // valid tokens of this warp's tile
      const uint32_t tile = ring_w + stage * S::TT;

      uint32_t kw[S::KWT], sw[S::SW], vw[S::VWT];
      load_lane_words<S::KWT>(tile + S::OFF_KC, lane, kw);
      load_lane_words<S::SW>(tile + S::OFF_KS, lane, sw);
      load_lane_words<S::VWT>(tile + S::OFF_VC, lane, vw);
      const uint2 ksc = lds_ring64(tile + S::OFF_KSC + gid * 8);
      const uint32_t vsc = lds_ring32(tile + S::OFF_VSC + gid * 4);

      // ---- cold logits: polar part, (A_hi + A_lo) . (q'_hi + q'_lo) ------
      // k-steps accumulate round-robin into kAccSplit chains
      float c1[kAccSplit][4] = {}, c2[kAccSplit][4] = {};
#pragma unroll
      for (int s = 0; s < S::NT; ++s) {
        const uint32_t o0 = lut_offset<BW, 7>(kw, (2 * s) * BW, lane_lut);
        const uint32_t o1 = lut_offset<BW, 7>(kw, (S::PT + 2 * s) * BW, lane_lut);
        const uint32_t o2 = lut_offset<BW, 7>(kw, (2 * s + 1) * BW, lane_lut);
        const uint32_t o3 = lut_offset<BW, 7>(kw, (S::PT + 2 * s + 1) * BW, lane_lut);
        const uint2 a0 = make_uint2(lut_hi(o0), lut_lo(o0));
        const uint2 a1 = make_uint2(lut_hi(o1), lut_lo(o1));
        const uint2 a2 = make_uint2(lut_hi(o2), lut_lo(o2));
        const uint2 a3 = make_uint2(lut_hi(o3), lut_lo(o3));
        mma16816(c1[s % kAccSplit], a0.x, a1.x, a2.x, a3.x, bq[s][0], bq[s][1]);
        if constexpr (PACK) {
          mma16816(c1[s % kAccSplit], a0.y, a1.y, a2.y, a3.y, bq[s][0], bq[s][1]);
        } else {
          mma16816(c2[s % kAccSplit], a0.x, a1.x, a2.x, a3.x, bq2[s][0], bq2[s][1]);
          mma16816(c2[s % kAccSplit], a0.y, a1.y, a2.y, a3.y, bq[s][0], bq[s][1]);
        }
      }
      // ---- cold logits: QJL part ---------------------------------------
      uint32_t x0, x1;
      if constexpr (M == 128) {
        x0 = sw[0];
        x1 = sw[S::SW - 1];
      } else {
        x0 = spread16(sw[0] & 0xffffu);
        x1 = spread16(sw[0] >> 16);
      }
      float cq0[4] = {0.f, 0.f, 0.f, 0.f}, cq1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < S::QS; s += 2) {
        mma16816(cq0, sign_pair(x0, 2 * s), sign_pair(x1, 2 * s), sign_pair(x0, 2 * s + 1),
                 sign_pair(x1, 2 * s + 1), qs[s][0], qs[s][1]);
        mma16816(cq1, sign_pair(x0, 2 * s + 2), sign_pair(x1, 2 * s + 2), sign_pair(x0, 2 * s + 3),
                 sign_pair(x1, 2 * s + 3), qs[s + 1][0], qs[s + 1][1]);
      }

      const bool v0 = gid < nvalid, v1 = gid + 8 < nvalid;
      const float sk0 = __half2float(__ushort_as_half((unsigned short)(ksc.x & 0xffffu)));
      const float sk1 = __half2float(__ushort_as_half((unsigned short)(ksc.x >> 16)));
      const float rn0 = __half2float(__ushort_as_half((unsigned short)(ksc.y & 0xffffu)));
      const float rn1 = __half2float(__ushort_as_half((unsigned short)(ksc.y >> 16)));
      float cp[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cp[j] = c1[0][j] + c2[0][j];
#pragma unroll
        for (int k = 1; k < kAccSplit; ++k) cp[j] += c1[k][j] + c2[k][j];
      }
      // entry j: token gid + 8 (j / HPL), head j % HPL
      float l2[2 * HPL];
      if constexpr (PACK) {       // columns 2 tig (hi) and 2 tig + 1 (lo) of head tig
        l2[0] = v0 ? fmaf(rn0 * kqjl[0], cq0[0] + cq1[0], sk0 * kpol[0] * (cp[0] + cp[1])) : kNegInf;
        l2[1] = v1 ? fmaf(rn1 * kqjl[0], cq0[2] + cq1[2], sk1 * kpol[0] * (cp[2] + cp[3])) : kNegInf;
      } else {
        l2[0] = v0 ? fmaf(rn0 * kqjl[0], cq0[0] + cq1[0], sk0 * kpol[0] * cp[0]) : kNegInf;
        l2[1] = v0 ? fmaf(rn0 * kqjl[1], cq0[1] + cq1[1], sk0 * kpol[1] * cp[1]) : kNegInf;
        l2[2] = v1 ? fmaf(rn1 * kqjl[0], cq0[2] + cq1[2], sk1 * kpol[0] * cp[2]) : kNegInf;
        l2[3] = v1 ? fmaf(rn1 * kqjl[1], cq0[3] + cq1[3], sk1 * kpol[1] * cp[3]) : kNegInf;
      }
      // V weights of tokens past the end are 0 (their records are not written)
      const float sv0 = v0 ? __half2float(__ushort_as_half((unsigned short)(vsc & 0xffffu))) : 0.f;
      const float sv1 = v1 ? __half2float(__ushort_as_half((unsigned short)(vsc >> 16))) : 0.f;
      float pv[2 * HPL];
      softmax_step(st, l2, sv0, sv1, pv);
      uint32_t pb0, pb1;
      pv_fragments<HPL>(pv, pb0, pb1);

      // ---- P V: V codes of pairs PV*gid + j for tokens 2tig, 2tig+1, +8, +9
#pragma unroll
      for (int j = 0; j < S::NT; ++j) {
        const uint32_t L0 = lut_hi(lut_offset<BW, 7>(vw, (0 * S::PV + j) * BW, lane_lut));
        const uint32_t L1 = lut_hi(lut_offset<BW, 7>(vw, (1 * S::PV + j) * BW, lane_lut));
        const uint32_t L2 = lut_hi(lut_offset<BW, 7>(vw, (2 * S::PV + j) * BW, lane_lut));
        const uint32_t L3 = lut_hi(lut_offset<BW, 7>(vw, (3 * S::PV + j) * BW, lane_lut));
        mma16816(st.O[j], __byte_perm(L0, L1, 0x5410), __byte_perm(L0, L1, 0x7632),
                 __byte_perm(L2, L3, 0x5410), __byte_perm(L2, L3, 0x7632), pb0, pb1);
      }
      }   // tile compute
      // ---- refill the stage with this warp's tile of block i + NS --------
      __syncwarp();
      if (lane == 0 && !aborted && i + S::NS < nblk) {
        fence_proxy_async();
        fetch_next(stage);
      }
    }
    __syncthreads();
    if (*abort_flag) {
      // A bulk copy did not complete in time: latch the error, give the
      // copies still in flight a bounded chance to land, and leave.
      if (tid == 0) atomicOr(a.status, kStatusTimeout);
      if (lane == 0)             // stage s received copies s, s + NS, ...: wait for its last one
        for (int s = 0; s < S::NS && s < issued; ++s) {
          const int n_s = (issued - s + S::NS - 1) / S::NS;
          mbar_wait_bounded(bar_w + 8 * s, (uint32_t)((n_s - 1) & 1));
        }
      return;
    }
    // with PACK, lanes tig >= 2 duplicate the heads of lanes tig - 2;
    // flush_partial keeps head 2 * tig + hh < G <= 4 only, i.e. tig < 2
    if (unit_cur >= 0) {
      flush_partial<D, S::NT, HPL>(st, false, inv_levels, G, merge,
                              a.part + (((size_t)(GATE ? uid_cur : unit_cur) * slots + slot_cur) * G) * (D + 2));
      st.reset();
    }
  }
  if (c < pl.hot_ctas) {
    // ====== then hot tiles [c * tpc, (c + 1) * tpc): the ring is idle ======
    const int ht = pl.hot_tiles;
    const int64_t total = (int64_t)a.units * ht;
    const int64_t f_lo = (int64_t)c * pl.hot_tpc;
    const int64_t f_hi = f_lo + pl.hot_tpc < total ? f_lo + pl.hot_tpc : total;
    constexpr int CH = D / 8;        // 16-byte chunks per token row
    WarpState<S::NT, 2> sh;          // hot logits use one MMA column per head
    sh.reset();
    uint32_t qh[S::NT][2];
    int unit_cur = -1, slot_cur = 0;
    int unit = (int)(f_lo / ht);
    int tile = (int)(f_lo - (int64_t)unit * ht);
    for (int64_t f = f_lo; f < f_hi; ++f, ++tile) {
      if (tile == ht) {
        tile = 0;
        ++unit;
      }
      if (unit != unit_cur) {
        if (unit_cur >= 0) {
          flush_partial<D, S::NT, 2>(sh, true, inv_levels, G, merge,
                                  a.part + (((size_t)unit_cur * slots + slot_cur) * G) * (D + 2));
          sh.reset();
        }
        unit_cur = unit;
        slot_cur = pl.slots_cold + (c - (int)(((int64_t)unit * ht) / pl.hot_tpc));
        const int b = unit / a.Hkv, kvh = unit % a.Hkv;
        const int head0 = b * a.Hq + kvh * G;
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
      }
      // the tile's K rows, then (in the same buffer) its V rows
      auto stage_rows = [&](const __half* src) {
        __syncthreads();
        for (int i = tid; i < S::TB * CH; i += kThreads) {
          const int r = i / CH, cc = i % CH;
          const int slot = tile * S::TB + r;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (slot < a.n_hot)
            v = __ldg(reinterpret_cast<const uint4*>(src + ((size_t)unit * a.W + slot) * D) + cc);
          *reinterpret_cast<uint4*>(ring + r * S::RS + cc * 16) = v;
        }
        __syncthreads();
      };
      const int nvalid = a.n_hot - tile * S::TB < S::TB ? a.n_hot - tile * S::TB : S::TB;
      const bool live = tb < nvalid;
      const uint32_t base = smem_addr(ring);
      const int mi = lane >> 3, rr = lane & 7;
      stage_rows(a.hot_k);
      uint32_t pb0 = 0u, pb1 = 0u;
      if (live) {
        float cc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < S::NT; ++s) {
          uint32_t af[4];
          ldsm_x4(af, base + (tb + rr + (mi & 1) * 8) * S::RS + (16 * s + (mi >> 1) * 8) * 2);
          mma16816(cc4, af[0], af[1], af[2], af[3], qh[s][0], qh[s][1]);
        }
        const bool v0 = tb + gid < nvalid, v1 = tb + gid + 8 < nvalid;
        float l2[4];
        l2[0] = v0 ? a.log2e_sigma * cc4[0] : kNegInf;
        l2[1] = v0 ? a.log2e_sigma * cc4[1] : kNegInf;
        l2[2] = v1 ? a.log2e_sigma * cc4[2] : kNegInf;
        l2[3] = v1 ? a.log2e_sigma * cc4[3] : kNegInf;
        float pv[4];
        softmax_step(sh, l2, 1.f, 1.f, pv);
        pv_fragments<2>(pv, pb0, pb1);
      }
      stage_rows(a.hot_v);
      if (live) {
#pragma unroll
        for (int j = 0; j < S::NT; ++j) {
          uint32_t af[4];
          ldsm_x4_trans(af, base + (tb + rr + (mi >> 1) * 8) * S::RS + (16 * j + (mi & 1) * 8) * 2);
          mma16816(sh.O[j], af[0], af[1], af[2], af[3], pb0, pb1);
        }
      }
    }
    if (unit_cur >= 0) {
      __syncthreads();
      flush_partial<D, S::NT, 2>(sh, true, inv_levels, G, merge,
                              a.part + (((size_t)unit_cur * slots + slot_cur) * G) * (D + 2));
    }
  }
}

// ---------------------------------------------------------------------------
// combine
// ---------------------------------------------------------------------------
// One block per query head, one thread per output dimension.  The split
// records' (m, l) pairs are read once by as many threads, so every global
// load of the block is independent of the others; R^T is applied to the
// cold sum with butterflies in registers (shuffles) and, for strides of a
// warp or more, through shared memory.
constexpr int kCombineMaxSlots = 128;

__global__ void combine_kernel(const CombineArgs a) {
  __shared__ float sw[kCombineMaxSlots];     // per-slot weight 2^(m_s - m)
  __shared__ float red[2][8];
  __shared__ float xbuf[256];
  // The next step's eviction encode may start its prologue now (it waits
  // for this kernel before reading its inputs).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int hg = blockIdx.x;
  const int b = hg / a.Hq, hq = hg % a.Hq;
  const int kvh = hq / a.G, g = hq % a.G;
  const int unit = b * a.Hkv + kvh;
  const int D = a.d, t = threadIdx.x, lane = t & 31, warp = t >> 5, nw = blockDim.x >> 5;
  const SplitPlan& pl = a.plan;
  const int slots = pl.slots_cold + pl.slots_hot;
  const float* base = a.part + (size_t)unit * slots * a.G * (D + 2);
  int nc = 0, nh = 0;
  if (pl.cold_ctas > 0 && pl.cold_blocks > 0) {
    const int64_t nb = pl.cold_blocks;
    if (a.unit_pos == nullptr) {
      nc = (int)(((unit + 1) * nb - 1) / pl.cold_bpc - (unit * nb) / pl.cold_bpc + 1);
    } else if (!a.head_skip[hg]) {       // gated: this head reads its unit's cold runs
      const int64_t p = a.unit_pos[unit];
      if (p >= 0) {
        int64_t bpc;
        int ctas;
        gated_cold_split(*a.n_active, nb, pl.cold_ctas, &bpc, &ctas);
        nc = (int)(((p + 1) * nb - 1) / bpc - (p * nb) / bpc + 1);
      }
    }
  }
  if (pl.hot_ctas > 0 && pl.hot_tiles > 0) {
    const int64_t ht = pl.hot_tiles;
    nh = (int)(((unit + 1) * ht - 1) / pl.hot_tpc - (unit * ht) / pl.hot_tpc + 1);
  }
  const int ns = nc + nh;
  auto rec = [&](int s) {
    return base + ((size_t)(s < nc ? s : pl.slots_cold + (s - nc)) * a.G + g) * (D + 2);
  };
  // ---- m = max over slots, then w_s and l = sum w_s l_s ----------------------
  float ms[kCombineMaxSlots / 64], ls[kCombineMaxSlots / 64];
  float mx = kNegInf;
#pragma unroll
  for (int k = 0; k < kCombineMaxSlots / 64; ++k) {
    const int s = t + k * blockDim.x;
    ms[k] = kNegInf;
    ls[k] = 0.f;
    if (s < ns) {
      const float* pp = rec(s);
      ms[k] = pp[0];
      ls[k] = pp[1];
    }
    mx = fmaxf(mx, ms[k]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
  if (lane == 0) red[0][warp] = mx;
  __syncthreads();
  mx = red[0][0];
  for (int w = 1; w < nw; ++w) mx = fmaxf(mx, red[0][w]);
  float lsum = 0.f;
#pragma unroll
  for (int k = 0; k < kCombineMaxSlots / 64; ++k) {
    const int s = t + k * blockDim.x;
    if (s < ns) {
      const float w = ms[k] == kNegInf ? 0.f : exp2f(ms[k] - mx);
      sw[s] = w;
      lsum += w * ls[k];
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(kFull, lsum, o);
  if (lane == 0) red[1][warp] = lsum;
  __syncthreads();
  lsum = 0.f;
  for (int w = 0; w < nw; ++w) lsum += red[1][w];
  // ---- weighted sums of the o vectors (independent loads) --------------------
  float oc = 0.f, oh = 0.f;
  if (mx != kNegInf) {
#pragma unroll 8
    for (int s = 0; s < nc; ++s) oc += sw[s] * rec(s)[2 + t];
#pragma unroll 4
    for (int s = nc; s < ns; ++s) oh += sw[s] * rec(s)[2 + t];
  }
  // ---- R^T on the cold sum: unnormalised Hadamard, then signs / sqrt(d) ------
  float x = oc;
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const float o = __shfl_xor_sync(kFull, x, h);
    x = (t & h) ? (o - x) : (x + o);
  }
  for (int h = 32; h < D; h <<= 1) {
    xbuf[t] = x;
    __syncthreads();
    const float o = xbuf[t ^ h];
    __syncthreads();
    x = (t & h) ? (o - x) : (x + o);
  }
  const float res = mx == kNegInf ? 0.f
                                  : (oh + (float)a.signs[t] * x * rsqrtf((float)D)) / lsum;
  a.out[(size_t)hg * D + t] = res;
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
typedef void (*AttendFn)(const AttendArgs);

template <int D, int M, int BW>
AttendFn attend_fn(bool pack, bool gate, int* smem) {
  *smem = AttendShape<D, M, BW>::SMEM;
  if (gate) return pack ? attend_kernel<D, M, BW, true, true> : attend_kernel<D, M, BW, false, true>;
  return pack ? attend_kernel<D, M, BW, true, false> : attend_kernel<D, M, BW, false, false>;
}

template <int D, int M>
AttendFn pick_bw(int bw, bool pack, bool gate, int* smem) {
  switch (bw) {
    case 2: return attend_fn<D, M, 2>(pack, gate, smem);
    case 3: return attend_fn<D, M, 3>(pack, gate, smem);
    case 4: return attend_fn<D, M, 4>(pack, gate, smem);
    case 5: return attend_fn<D, M, 5>(pack, gate, smem);
    case 6: return attend_fn<D, M, 6>(pack, gate, smem);
    case 7: return attend_fn<D, M, 7>(pack, gate, smem);
    case 8: return attend_fn<D, M, 8>(pack, gate, smem);
  }
  return nullptr;
}

// groups of up to 4 query heads use the packed [q'_hi | q'_lo] columns
AttendFn pick_attend(const Layout& L, int G, bool gate, int* smem) {
  const bool pack = G <= 4;
  if (L.d == 64 && L.m == 64) return pick_bw<64, 64>(L.bw, pack, gate, smem);
  if (L.d == 64 && L.m == 128) return pick_bw<64, 128>(L.bw, pack, gate, smem);
  if (L.d == 128 && L.m == 64) return pick_bw<128, 64>(L.bw, pack, gate, smem);
  if (L.d == 128 && L.m == 128) return pick_bw<128, 128>(L.bw, pack, gate, smem);
  return nullptr;
}

}  // namespace

int attend_ctas_per_sm(const Layout& L, int G) {
  int smem = 0;
  AttendFn fn = pick_attend(L, G, false, &smem);
  AttendFn fg = pick_attend(L, G, true, &smem);
  if (!fn || !fg) return 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(fg, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem) != cudaSuccess) return 0;
  return n;
}

template <int D, int M>
cudaError_t launch_qprep_dm(const QPrepArgs& a, cudaStream_t s) {
  const int grid = (a.heads + 256 / M - 1) / (256 / M);
  constexpr int smem = D * M * 4;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(qprep_kernel<D, M>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  // Programmatic dependent launch: q-prep reads only the query and S^T,
  // so it may overlap the kernel before it (the eviction encode); it waits
  // for that kernel before it exits, so work after q-prep still finds the
  // encode complete.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qprep_kernel<D, M>, a);
}

cudaError_t launch_qprep(const QPrepArgs& a, cudaStream_t s) {
  if (a.d == 64 && a.m == 64) return launch_qprep_dm<64, 64>(a, s);
  if (a.d == 64 && a.m == 128) return launch_qprep_dm<64, 128>(a, s);
  if (a.d == 128 && a.m == 64) return launch_qprep_dm<128, 64>(a, s);
  if (a.d == 128 && a.m == 128) return launch_qprep_dm<128, 128>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
  int smem = 0;
  AttendFn fn = pick_attend(a.L, a.G, a.alist != nullptr, &smem);
  if (!fn) return cudaErrorInvalidValue;
  const int grid = a.plan.cold_ctas > a.plan.hot_ctas ? a.plan.cold_ctas : a.plan.hot_ctas;
  if (grid == 0) return cudaSuccess;
  fn<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  combine_kernel<<<a.batch * a.Hq, a.d, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
