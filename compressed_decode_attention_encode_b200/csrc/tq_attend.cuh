// The decode-attention kernel over the packed cold cache and the fp16 hot
// ring ("TurboQuant: optimización de memoria para KV caches en inferencia de
// LLMs", flow step 6: attention logits from the compressed cache; "Monarch
// v3 ...", "Bucle de Decodificación Simplificado": aggregate the hot and
// cold scores, softmax, apply).  Included by the per-shape instantiation
// files tq_attend_<d>_<m>.cu, so that the shapes compile in parallel.
//
// One wave of CTAs.  Cold CTAs take equal contiguous runs of the flattened
// (unit, 64-token block) list; each warp streams its own 16-token tile of
// every block through an NS-stage shared-memory ring filled by
// cp.async.bulk (mbarrier completion, bounded waits).  Per tile:
//   key logits, polar part   [16 tok x pairs] . q'
//     SLOT (b_theta <= 3): a pair's unit reconstruction c_r (cos, sin)(th)
//       is exactly c_r * (+-1) times one of S = 2^(b_theta-1) directions
//       e(pi k / S); one table lookup gives the pair's 4 int8 slots
//       (c_r * sign in slot k), and the query side holds the projections
//       <q'_pair, e(pi k / S)> as two int8 planes: an exact int8 MMA
//       (m16n8k32, int32 accumulation) per 8 pairs.
//     HILO (b_theta >= 4): fp16 tables of c_r (cos, sin) as hi + lo parts
//       against q' as fp16 hi + lo (m16n8k16, fp32 accumulation).
//   key logits, QJL part     [16 tok x m] . q'': the sign bits become 0/1
//       bytes with one shift and one mask per 4 bits; q'' enters as two int8
//       planes; sum_i q''_i (2 b_i - 1) = 2 sum_i b_i q''_i - sum_i q''_i.
//   P V                      [d x 16 tok] . P: fp16 table of the values'
//       unit pairs, P transposed in registers with movmatrix.
// with an online softmax (exp2 domain).  Hot CTAs stream fp16 tiles
// through padded shared memory (ldmatrix).
#pragma once

#include <cfloat>
#include <type_traits>

#include "tq_internal.cuh"

namespace tq {
namespace att {

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

// ---- PTX helpers -----------------------------------------------------------
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// int8 x int8 -> int32, 16 x 8 x 32.  A row-major (a0: row gid, k 4 tig..;
// a1: row gid + 8; a2, a3: k + 16), B column-major (b0: column gid, k
// 4 tig..; b1: k + 16), C rows gid / gid + 8, columns 2 tig, 2 tig + 1.
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with a zero accumulator in (the first k-step of a product).
__device__ __forceinline__ void mma_s8_z(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};\n"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
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

// try_wait that may suspend the thread (issuing nothing) until the phase
// completes or about 1 ms has passed.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of an mbarrier, giving up after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait_suspend(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 0/1 bytes from the sign bits sh, sh + 8, sh + 16, sh + 24 of x.
__device__ __forceinline__ uint32_t sign_bytes(uint32_t x, int sh) {
  return (x >> sh) & 0x01010101u;
}

// Byte offset in a LUT whose entries are 2^SH bytes apart, of the entry
// named by the BW-bit field at bit `pos` of the lane's word stream (`pos`
// is a compile-time constant after unrolling), plus `lane_off` (the lane's
// copy inside the entry): one shift (a funnel shift for a field straddling
// two words) and one three-input logic op.
template <int BW, int SH, int NW>
__device__ __forceinline__ uint32_t lut_offset(const uint32_t (&w)[NW], int pos, uint32_t lane_off) {
  constexpr uint32_t kMask = ((1u << BW) - 1u) << SH;
  const int wi = pos >> 5, bi = pos & 31;
  uint32_t t, r;
  if (bi + BW <= 32 || wi + 1 >= NW) {
    if (bi > SH) asm("shr.b32 %0, %1, %2;" : "=r"(t) : "r"(w[wi]), "r"(bi - SH));
    else if (bi == SH) t = w[wi];
    else t = w[wi] << (SH - bi);
  } else {
    asm("shf.r.wrap.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(w[wi]), "r"(w[wi + 1]), "r"(bi - SH));
  }
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(t), "n"(kMask), "r"(lane_off));   // (t & m) | l
  return r;
}

// Table lookups at a lane offset (+ a compile-time table offset).
template <int OFF>
__device__ __forceinline__ uint32_t lut_at(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}

// ---------------------------------------------------------------------------
// Shape constants of one instantiation.
// ---------------------------------------------------------------------------
template <int D, int M, int BW>
struct AttendShape {
  static constexpr int P = D / 2;
  static constexpr int NT = D / 16;                 // K k-steps (8 pairs each) == PV m-tiles
  static constexpr int QS = M / 32;                 // k-steps of the int8 QJL product
  static constexpr int PT = P / 4;                  // K pairs per lane (per token)
  static constexpr int KWT = (2 * PT * BW + 31) / 32;
  static constexpr int SW = (2 * (M / 4) + 31) / 32;
  static constexpr int VWT = KWT;                   // V codes: the K layout
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_KS = OFF_KC + 128 * KWT;
  static constexpr int OFF_KSC = OFF_KS + 128 * SW;
  static constexpr int OFF_VC = OFF_KSC + 64;
  static constexpr int OFF_VSC = OFF_VC + 128 * VWT;
  static constexpr int TT = OFF_VSC + 32;           // tile bytes
  static constexpr int TB = kTokensPerBlock;
  static constexpr int BLOCK = kTilesPerBlock * TT;
  static constexpr int NLUT = 1 << BW;
  // Two tables of 4-byte entries, one copy per lane per entry (entries 128
  // bytes apart): table A (SLOT: the keys' int8 slots; HILO: fp16 c_r
  // (cos, sin), keys and values), then table B (SLOT: the values' fp16
  // pairs; HILO: the keys' fp16 rounding remainders).  Table A starts on a
  // LUT_ALIGN boundary of the shared window, so a lookup's address is
  // (table | entry << 7 | lane << 2) -- one logic op -- and table B's entry
  // is the same address + LUT_BYTES.
  static constexpr int LUT_BYTES = NLUT * 32 * 4;
  static constexpr int LUT_ALIGN = 128 << BW;
  static constexpr int RS = 2 * D + 16;             // padded hot row stride (bytes)
  static constexpr int HOT_BYTES = TB * RS;          // one hot tile, K then V
  static constexpr int MERGE_BYTES = (64 + 8 * D) * 4;
  // up to 8 stages per warp: 4 x 8 barriers, the abort flag
  static constexpr int BAR_BYTES = 4 * 8 * 8 + 16;
  // Dynamic shared memory: [ring | pad | LUT A | LUT B | merge | barriers],
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

constexpr float kPvMax = 256.f;        // V weights p * s16_v stay <= 2^8 (fp16 operands)
constexpr float kPMax = 0x1p100f;      // softmax numerators p stay <= 2^100 (fp32 sums)
constexpr float kPRange = 100.f;

// Which query heads a lane (gid, tig) holds on the cold path: HMAP_PACK --
// head tig in both MMA columns 2 tig, 2 tig + 1 (groups of up to 4);
// HMAP_PAIR -- heads 2 tig + hh (HILO, groups of up to 8); HMAP_SPLIT --
// heads tig + 4 hh (SLOT, groups of 5 to 8: two int8 MMAs per k-step).
// Column 2 tig + hh of the PV product carries head number hh of the lane.
enum { HMAP_PACK = 0, HMAP_PAIR = 1, HMAP_SPLIT = 2 };

template <int HMAP>
__device__ __forceinline__ int lane_head(int tig, int hh) {
  if constexpr (HMAP == HMAP_PACK) return tig;
  else if constexpr (HMAP == HMAP_PAIR) return 2 * tig + hh;
  else return tig + 4 * hh;
}

// Per-warp softmax / accumulator state for one unit: the reference `ref`
// (log2 domain) of the numerators p = 2^(l - ref) summed in `l_run`, and
// the accumulators O of the V weights p * s16_v.  A lane holds HPL query
// heads (see lane_head).
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
// lane_head<HMAP>(tig, hh) (heads >= G are dropped).  Called by all threads
// of the CTA; uses the merge area: per-warp m / l, then per-warp o rows
// summed by the threads.
template <int D, int NT, int HPL, int HMAP>
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
  // (lanes whose head is >= G hold no head: their values are never used)
  if (gid == 0) {
#pragma unroll
    for (int hh = 0; hh < HPL; ++hh) {
      const int g = lane_head<HMAP>(tig, hh);
      mw[warp * 8 + g] = st.ref[hh];
      lw[warp * 8 + g] = st.l_run[hh];
    }
  }
  for (int i = tid; i < 8 * D; i += kThreads) ow[i] = 0.f;
  __syncthreads();
  float f[HPL];
#pragma unroll
  for (int hh = 0; hh < HPL; ++hh) {
    const int g = lane_head<HMAP>(tig, hh);
    float mx = kNegInf;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, mw[w * 8 + g]);
    f[hh] = st.ref[hh] == kNegInf ? 0.f : fast_exp2(st.ref[hh] - mx) * (hot ? 1.f : inv_levels);
  }
  constexpr int PT = D / 8;    // cold rows: pair (gid / 2) * PT + 2 i + r2, component gid % 2
  // the 4 warps add their rows in turn: no two threads touch one word at once
  for (int w = 0; w < 4; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < NT; ++i) {
#pragma unroll
        for (int r2 = 0; r2 < 2; ++r2) {
          const int dim = hot ? (16 * i + gid + 8 * r2) : (2 * ((gid >> 1) * PT + 2 * i + r2) + (gid & 1));
#pragma unroll
          for (int hh = 0; hh < HPL; ++hh) {
            const int g = lane_head<HMAP>(tig, hh);
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

// ---------------------------------------------------------------------------
// The kernel.  SLOT selects the int8 polar path (b_theta <= 3); HMAP the
// heads a lane holds on the cold path (HMAP_PACK for groups of up to 4;
// HMAP_SPLIT for larger SLOT groups, HMAP_PAIR for larger HILO groups);
// MODE: plain, gated (the cold tier of listed units only), with every
// cold token's logits written out (promotion), or ragged (per-row counts
// from a RowTable: the units' blocks and tiles are flattened by prefix
// sums, so rows of any length share the CTAs evenly).
// ---------------------------------------------------------------------------
enum { MODE_PLAIN = 0, MODE_GATED = 1, MODE_LOGITS = 2, MODE_RAGGED = 3 };

template <int D, int M, int BW, bool SLOT, int HMAP, int MODE>
__global__ void __launch_bounds__(kThreads, kAttendMinBlocks) attend_kernel(const AttendArgs a) {
  constexpr bool GATE = MODE == MODE_GATED;
  constexpr bool RAGGED = MODE == MODE_RAGGED;
  using S = AttendShape<D, M, BW>;
  constexpr int HPL = HMAP == HMAP_PACK ? 1 : 2;     // query heads per lane on the cold path
  constexpr int NQ = SLOT ? HPL : 1;                 // int8 MMAs per k-step (column groups)
  constexpr bool PACKQ = HMAP == HMAP_PACK;          // HILO: [q'_hi | q'_lo] packed columns
  static_assert(!(SLOT && HMAP == HMAP_PAIR) && !(!SLOT && HMAP == HMAP_SPLIT), "head map");
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* lut_a = reinterpret_cast<uint32_t*>(smem + S::OFF_LUT);
  uint32_t* lut_b = lut_a + S::NLUT * 32;
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
  const uint32_t lut_sa = smem_addr(lut_a);
  if (lut_sa & (S::LUT_ALIGN - 1)) {   // dynamic base not where the layout assumes
    if (tid == 0) atomicOr(a.status, kStatusLayout);
    return;
  }
  const uint32_t lane_lut = lut_sa | ((uint32_t)lane * 4u);   // this lane's copy, table A
  const SplitPlan& pl = a.plan;
  const int slots = pl.slots_cold + pl.slots_hot;
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
    // Positions of the run: units (gated: active-list positions), each with
    // pos_blocks(p) blocks starting at flattened block pos_off(p); ragged
    // runs skip the units of rows without cold tokens.
    const int n_rows = a.units / a.Hkv;
    auto row_blocks = [&](int b) -> int { return (a.rows->n_cold[b] + S::TB - 1) / S::TB; };
    auto pos_blocks = [&](int p) -> int {
      if constexpr (RAGGED) return row_blocks(p / a.Hkv); else return (int)pl.cold_blocks;
    };
    auto pos_off = [&](int p) -> int64_t {
      if constexpr (RAGGED) {
        const int b = p / a.Hkv;
        return a.rows->cold_pre[b] + (int64_t)(p % a.Hkv) * row_blocks(b);
      } else {
        return (int64_t)p * pl.cold_blocks;
      }
    };
    auto pos_tail = [&](int p) -> int {     // valid tokens of the position's last block
      if constexpr (RAGGED) return a.rows->n_cold[p / a.Hkv] - (pos_blocks(p) - 1) * S::TB;
      else return (int)(a.n_cold - (pl.cold_blocks - 1) * S::TB);
    };
    auto pos_next = [&](int p) -> int {
      if constexpr (RAGGED) {
        if ((p + 1) % a.Hkv != 0) return p + 1;
        int b = (p + 1) / a.Hkv;
        while (b < n_rows && a.rows->n_cold[b] == 0) ++b;
        return b * a.Hkv;
      } else {
        return p + 1;
      }
    };
    // (gated: alist[n_active] exists, so the run's last step may look one past)
    auto pos_uid = [&](int p) -> int { if constexpr (GATE) return a.alist[p]; else return p; };
    const int64_t total = RAGGED ? (int64_t)a.rows->cold_pre[n_rows] : cold_units() * pl.cold_blocks;
    const int64_t f_lo = (int64_t)c * cold_bpc();
    const int64_t f_hi = f_lo + cold_bpc() < total ? f_lo + cold_bpc() : total;
    const int nblk = (int)(f_hi - f_lo);
    int p_first, blk_first;
    if constexpr (RAGGED) {      // the row holding block f_lo: the last b with cold_pre[b] <= f_lo
      int lo = 0, hi = n_rows - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.rows->cold_pre[mid] <= f_lo) lo = mid; else hi = mid - 1;
      }
      const int nbr = row_blocks(lo);
      const int64_t off = f_lo - a.rows->cold_pre[lo];
      p_first = lo * a.Hkv + (int)(off / nbr);
      blk_first = (int)(off % nbr);
    } else {
      p_first = (int)(f_lo / pl.cold_blocks);
      blk_first = (int)(f_lo - (int64_t)p_first * pl.cold_blocks);
    }
    const uint32_t bar_w = smem_addr(bars) + 8 * S::NS * warp;           // this warp's barriers
    const uint32_t ring_w = smem_addr(ring) + S::NS * S::TT * warp;      // this warp's stages
    // The warp's tile stream: `nsrc` is the next tile to fetch (block
    // `nblk_b` of position `fpos`, which has `fnb` blocks); at a position's
    // end it moves to block 0 of the next one.  `issued` counts the copies.
    int fpos = p_first, nblk_b = blk_first, fnb = pos_blocks(p_first), issued = 0;
    const uint8_t* nsrc =
        a.cold + ((size_t)pos_uid(fpos) * a.L.blocks_per_unit + (size_t)nblk_b) * S::BLOCK + warp * S::TT;
    // The next tile into stage s: every lane advances the (warp-uniform)
    // stream; lane 0 alone arms the barrier and issues the copy, predicated
    // rather than branched around.  `after_reads` orders the warp's reads of
    // the stage's previous tile before the asynchronous write.
    auto fetch_next = [&](int s, bool after_reads) {
      const uint32_t bar = bar_w + 8 * s;
      asm volatile(
          "{\n .reg .pred p, f;\n setp.eq.u32 p, %0, 0;\n setp.ne.u32 f, %5, 0;\n"
          " and.pred f, f, p;\n"
          " @f fence.proxy.async.shared::cta;\n"
          " @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n"
          " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%3], [%4], %2, [%1];\n}\n"
          ::"r"(lane), "r"(bar), "r"(S::TT), "r"(ring_w + s * S::TT), "l"(nsrc), "r"((int)after_reads)
          : "memory");
      ++issued;
      nsrc += S::BLOCK;
      if (++nblk_b == fnb) {
        nblk_b = 0;
        fpos = pos_next(fpos);
        if (RAGGED && fpos >= a.units) return;    // the run's last block has been issued
        fnb = pos_blocks(fpos);
        nsrc = a.cold + (size_t)pos_uid(fpos) * a.L.blocks_per_unit * S::BLOCK + warp * S::TT;
      }
    };
    if (tid == 0) *abort_flag = 0;
    if (lane == 0) {
      for (int s = 0; s < S::NS; ++s) mbar_init(bar_w + 8 * s, 1);
      fence_barrier_init();
    }
    __syncwarp();
    for (int s = 0; s < S::NS && s < nblk; ++s) fetch_next(s, false);
    // Tables of the code words e = (c_r << b_theta) | c_theta, one copy per
    // lane (the merge area is free at this point for the 2^bw distinct
    // entries, built once each).
    {
      const int bt = a.L.b_theta;
      uint2* base = reinterpret_cast<uint2*>(merge);
      for (int e = tid; e < S::NLUT; e += kThreads) {
        const int cr = e >> bt, ct = e & ((1 << bt) - 1);
        double sn, cs;
        sincospi(2.0 * (double)ct / (double)(1 << bt), &sn, &cs);
        const float x = (float)((double)cr * cs), y = (float)((double)cr * sn);
        const __half hx = __float2half_rn(x), hy = __float2half_rn(y);
        const uint32_t hi = pack_h2(__half2float(hx), __half2float(hy));
        if constexpr (SLOT) {
          // direction k = c_theta mod ns (angle pi k / ns), sign - for the
          // upper half of the circle's code range
          const int ns = bt > 1 ? (1 << (bt - 1)) : 1;
          const int k = ct & (ns - 1);
          const int v = ct < ns ? cr : -cr;
          base[e] = make_uint2(((uint32_t)(v & 0xff)) << (8 * k), hi);
        } else {
          base[e] = make_uint2(hi, pack_h2(x - __half2float(hx), y - __half2float(hy)));
        }
      }
      __syncthreads();
      for (int i = tid; i < S::NLUT * 32; i += kThreads) {
        const uint2 e = base[i >> 5];
        lut_a[i] = e.x;
        lut_b[i] = e.y;
      }
    }
    __syncthreads();

    // B operands, loaded per unit:
    //   SLOT  bk[nq][s]: the two int8 planes' projections of q' (column
    //         2 t + pl: plane pl of head lane_head(t, nq)); bs[nq][s]:
    //         those of q''
    //   HILO  bq[s]: q'_hi / q'_lo (packed: even / odd column of each head),
    //         bq2[s]: q'_lo when not packed; bs as SLOT
    constexpr int NQS = HPL;             // int8 column groups of the QJL product
    constexpr int kAccSplit = 2;         // independent accumulator chains
    uint32_t bk[SLOT ? NQ : 1][SLOT ? S::NT : 1][2];
    uint32_t bq[SLOT ? 1 : S::NT][2], bq2[(SLOT || PACKQ) ? 1 : S::NT][2];
    uint32_t bs[NQS][S::QS][2];
    float kpol[HPL], kqjl[HPL];
    int qsum[HPL];
    const bool forced_timeout = a.wait_limit_ns == 0;
    bool aborted = false;

    // Loads the B operands and logit constants of unit position `u`.
    auto setup_unit = [&](int u) {
      const int uid = pos_uid(u);
      const int b = uid / a.Hkv, kvh = uid % a.Hkv;
      const int head0 = b * a.Hq + kvh * G;
#pragma unroll
      for (int nq = 0; nq < NQS; ++nq) {
        const int hc = lane_head<HMAP>(gid >> 1, nq), pln = gid & 1;
        const bool live = hc < G;
        const uint2* qs = reinterpret_cast<const uint2*>(a.qs8 + ((size_t)(head0 + hc) * 2 + pln) * S::QS * 32) + tig;
#pragma unroll
        for (int s = 0; s < S::QS; ++s) {
          const uint2 v = live ? qs[4 * s] : make_uint2(0u, 0u);
          bs[nq][s][0] = v.x;
          bs[nq][s][1] = v.y;
        }
        if constexpr (SLOT) {
          const uint2* qk = reinterpret_cast<const uint2*>(a.qk8 + ((size_t)(head0 + hc) * 2 + pln) * S::NT * 32) + tig;
#pragma unroll
          for (int s = 0; s < S::NT; ++s) {
            const uint2 v = live ? qk[4 * s] : make_uint2(0u, 0u);
            bk[nq][s][0] = v.x;
            bk[nq][s][1] = v.y;
          }
        }
      }
      if constexpr (!SLOT) {
        // B column gid: head gid (8 heads) or, packed, head gid / 2 with
        // column parity 0 = q'_hi, 1 = q'_lo (the A_lo product uses the
        // even columns only)
        const int hcol = PACKQ ? (gid >> 1) : gid;
        const bool odd = PACKQ && (gid & 1);
        if (hcol < G) {
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.qrot + (size_t)(head0 + hcol) * 2 * D) + S::PT * tig;
          const int o1 = odd ? S::P : 0;
#pragma unroll
          for (int s = 0; s < S::NT; ++s) {
            bq[s][0] = qp[o1 + 2 * s];
            bq[s][1] = qp[o1 + 2 * s + 1];
            if constexpr (!PACKQ) {
              bq2[s][0] = qp[S::P + 2 * s];
              bq2[s][1] = qp[S::P + 2 * s + 1];
            }
          }
        } else {
#pragma unroll
          for (int s = 0; s < S::NT; ++s) bq[s][0] = bq[s][1] = 0u;
          if constexpr (!PACKQ) {
#pragma unroll
            for (int s = 0; s < S::NT; ++s) bq2[s][0] = bq2[s][1] = 0u;
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < HPL; ++hh) {
        const int g = lane_head<HMAP>(tig, hh);
        const float* qsc = a.qscale + 4 * (size_t)(head0 + g);
        const bool live = g < G;
        kpol[hh] = live ? a.log2e_sigma * (SLOT ? qsc[1] : qsc[0]) * inv_levels : 0.f;
        kqjl[hh] = live ? a.log2e_sigma * kSqrtHalfPi / (float)M * qsc[2] : 0.f;
        qsum[hh] = live ? __float_as_int(qsc[3]) : 0;
      }
      return uid;
    };

    // One 16-token tile of block i (stage i % NS of the warp's ring): wait
    // for its copy, compute, refill the stage with block i + NS.  MASKED
    // tiles (a unit's last block) hold `nvalid` < 16 valid tokens.
    auto tile_step = [&](int i, auto masked, int nvalid, int uid, int64_t tok0) {
      constexpr bool MASKED = decltype(masked)::value;
      const int stage = i % S::NS;         // NS need not be a power of two
      if (!aborted) {
        const bool got = !forced_timeout &&
                         mbar_wait_bounded(bar_w + 8 * stage, (uint32_t)((i / S::NS) & 1), a.wait_limit_ns);
        if (!__all_sync(kFull, got)) {
          aborted = true;
          if (lane == 0) *abort_flag = 1;
        }
      }
      if (!aborted && (!MASKED || nvalid > 0)) {
      const uint32_t tile = ring_w + stage * S::TT;

      uint32_t kw[S::KWT], sw[S::SW], vw[S::VWT];
      load_lane_words<S::KWT>(tile + S::OFF_KC, lane, kw);
      load_lane_words<S::SW>(tile + S::OFF_KS, lane, sw);
      load_lane_words<S::VWT>(tile + S::OFF_VC, lane, vw);
      const uint2 ksc = lds_ring64(tile + S::OFF_KSC + gid * 8);
      const uint32_t vsc = lds_ring32(tile + S::OFF_VSC + gid * 4);

      // ---- QJL part: 0/1 sign bytes (bit 8e + 2s + hf of the token's word;
      // for m = 64 the two tokens share one word, token gid + 8 at +4) ------
      int cq[NQS][4];
#pragma unroll
      for (int s = 0; s < S::QS; ++s) {
        uint32_t r0, r1, r2, r3;
        if constexpr (M == 128) {
          r0 = sign_bytes(sw[0], 2 * s);
          r1 = sign_bytes(sw[1], 2 * s);
          r2 = sign_bytes(sw[0], 2 * s + 1);
          r3 = sign_bytes(sw[1], 2 * s + 1);
        } else {
          r0 = sign_bytes(sw[0], 2 * s);
          r1 = sign_bytes(sw[0], 4 + 2 * s);
          r2 = sign_bytes(sw[0], 2 * s + 1);
          r3 = sign_bytes(sw[0], 4 + 2 * s + 1);
        }
#pragma unroll
        for (int nq = 0; nq < NQS; ++nq) {
          if (s == 0) mma_s8_z(cq[nq], r0, r1, r2, r3, bs[nq][s][0], bs[nq][s][1]);
          else mma_s8(cq[nq], r0, r1, r2, r3, bs[nq][s][0], bs[nq][s][1]);
        }
      }

      const bool v0 = !MASKED || gid < nvalid, v1 = !MASKED || gid + 8 < nvalid;
      const float sk0 = __half2float(__ushort_as_half((unsigned short)(ksc.x & 0xffffu)));
      const float sk1 = __half2float(__ushort_as_half((unsigned short)(ksc.x >> 16)));
      const float rn0 = __half2float(__ushort_as_half((unsigned short)(ksc.y & 0xffffu)));
      const float rn1 = __half2float(__ushort_as_half((unsigned short)(ksc.y >> 16)));
      // integer QJL sums of the lane's heads: 2 sum b q'' - sum q'' (two planes)
      float qj[2][HPL];
#pragma unroll
      for (int hh = 0; hh < HPL; ++hh) {       // group hh, columns 2 tig (hi), 2 tig + 1 (lo)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          qj[j][hh] = (float)(2 * (256 * cq[hh][2 * j] + cq[hh][2 * j + 1]) - qsum[hh]);
        }
      }
      // entry j: token gid + 8 (j / HPL), head j % HPL
      float l2[2 * HPL];
      if constexpr (SLOT) {
        // ---- polar part: int8 slots . projection planes ------------------
        int ck[NQ][4];
#pragma unroll
        for (int s = 0; s < S::NT; ++s) {
          const uint32_t o0 = lut_offset<BW, 7>(kw, (2 * s) * BW, lane_lut);
          const uint32_t o1 = lut_offset<BW, 7>(kw, (S::PT + 2 * s) * BW, lane_lut);
          const uint32_t o2 = lut_offset<BW, 7>(kw, (2 * s + 1) * BW, lane_lut);
          const uint32_t o3 = lut_offset<BW, 7>(kw, (S::PT + 2 * s + 1) * BW, lane_lut);
          const uint32_t a0 = lut_at<0>(o0), a1 = lut_at<0>(o1), a2 = lut_at<0>(o2), a3 = lut_at<0>(o3);
#pragma unroll
          for (int nq = 0; nq < NQ; ++nq) {
            if (s == 0) mma_s8_z(ck[nq], a0, a1, a2, a3, bk[nq][s][0], bk[nq][s][1]);
            else mma_s8(ck[nq], a0, a1, a2, a3, bk[nq][s][0], bk[nq][s][1]);
          }
        }
#pragma unroll
        for (int hh = 0; hh < HPL; ++hh) {
          const int p0 = 256 * ck[hh][0] + ck[hh][1];
          const int p1 = 256 * ck[hh][2] + ck[hh][3];
          l2[hh] = v0 ? fmaf(rn0 * kqjl[hh], qj[0][hh], sk0 * kpol[hh] * (float)p0) : kNegInf;
          l2[HPL + hh] = v1 ? fmaf(rn1 * kqjl[hh], qj[1][hh], sk1 * kpol[hh] * (float)p1) : kNegInf;
        }
      } else {
        // ---- polar part: (A_hi + A_lo) . (q'_hi + q'_lo) in fp16 ----------
        float c1[kAccSplit][4] = {}, c2[kAccSplit][4] = {};
#pragma unroll
        for (int s = 0; s < S::NT; ++s) {
          const uint32_t o0 = lut_offset<BW, 7>(kw, (2 * s) * BW, lane_lut);
          const uint32_t o1 = lut_offset<BW, 7>(kw, (S::PT + 2 * s) * BW, lane_lut);
          const uint32_t o2 = lut_offset<BW, 7>(kw, (2 * s + 1) * BW, lane_lut);
          const uint32_t o3 = lut_offset<BW, 7>(kw, (S::PT + 2 * s + 1) * BW, lane_lut);
          const uint2 a0 = make_uint2(lut_at<0>(o0), lut_at<S::LUT_BYTES>(o0));
          const uint2 a1 = make_uint2(lut_at<0>(o1), lut_at<S::LUT_BYTES>(o1));
          const uint2 a2 = make_uint2(lut_at<0>(o2), lut_at<S::LUT_BYTES>(o2));
          const uint2 a3 = make_uint2(lut_at<0>(o3), lut_at<S::LUT_BYTES>(o3));
          mma16816(c1[s % kAccSplit], a0.x, a1.x, a2.x, a3.x, bq[s][0], bq[s][1]);
          if constexpr (PACKQ) {
            mma16816(c1[s % kAccSplit], a0.y, a1.y, a2.y, a3.y, bq[s][0], bq[s][1]);
          } else {
            mma16816(c2[s % kAccSplit], a0.x, a1.x, a2.x, a3.x, bq2[s][0], bq2[s][1]);
            mma16816(c2[s % kAccSplit], a0.y, a1.y, a2.y, a3.y, bq[s][0], bq[s][1]);
          }
        }
        float cp[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cp[j] = c1[0][j] + c2[0][j] + c1[1][j] + c2[1][j];
        if constexpr (PACKQ) {     // columns 2 tig (hi) and 2 tig + 1 (lo) of head tig
          l2[0] = v0 ? fmaf(rn0 * kqjl[0], qj[0][0], sk0 * kpol[0] * (cp[0] + cp[1])) : kNegInf;
          l2[1] = v1 ? fmaf(rn1 * kqjl[0], qj[1][0], sk1 * kpol[0] * (cp[2] + cp[3])) : kNegInf;
        } else {
          l2[0] = v0 ? fmaf(rn0 * kqjl[0], qj[0][0], sk0 * kpol[0] * cp[0]) : kNegInf;
          l2[1] = v0 ? fmaf(rn0 * kqjl[1], qj[0][1], sk0 * kpol[1] * cp[1]) : kNegInf;
          l2[2] = v1 ? fmaf(rn1 * kqjl[0], qj[1][0], sk1 * kpol[0] * cp[2]) : kNegInf;
          l2[3] = v1 ? fmaf(rn1 * kqjl[1], qj[1][1], sk1 * kpol[1] * cp[3]) : kNegInf;
        }
      }
      if constexpr (MODE == MODE_LOGITS) {     // promotion: every valid token's logits
#pragma unroll
        for (int hh = 0; hh < HPL; ++hh) {
          const int g = lane_head<HMAP>(tig, hh);
          float* lp = a.logits + ((size_t)uid * a.logit_capacity + tok0 + gid) * G + g;
          if (g < G && v0) lp[0] = l2[hh];
          if (g < G && v1) lp[8 * G] = l2[HPL + hh];
        }
      }
      // V weights of tokens past the end are 0 (their records are not written)
      const float sv0 = v0 ? __half2float(__ushort_as_half((unsigned short)(vsc & 0xffffu))) : 0.f;
      const float sv1 = v1 ? __half2float(__ushort_as_half((unsigned short)(vsc >> 16))) : 0.f;
      float pv[2 * HPL];
      softmax_step(st, l2, sv0, sv1, pv);
      uint32_t pb0, pb1;
      pv_fragments<HPL>(pv, pb0, pb1);

      // ---- P V: m-tile j's rows are the 4 lanes' pairs tig*PT + 2j (rows
      // 0-7) and tig*PT + 2j + 1 (rows 8-15).  A lane's lookup of its pair
      // of token gid (gid + 8) is row gid of an 8x8 [token x dim] fragment;
      // movmatrix transposes it into the [dim x token] A fragment.
      constexpr int VOFF = SLOT ? S::LUT_BYTES : 0;    // the values' fp16 table
#pragma unroll
      for (int j = 0; j < S::NT; ++j) {
        const uint32_t L0 = lut_at<VOFF>(lut_offset<BW, 7>(vw, (2 * j) * BW, lane_lut));
        const uint32_t L1 = lut_at<VOFF>(lut_offset<BW, 7>(vw, (2 * j + 1) * BW, lane_lut));
        const uint32_t L2 = lut_at<VOFF>(lut_offset<BW, 7>(vw, (S::PT + 2 * j) * BW, lane_lut));
        const uint32_t L3 = lut_at<VOFF>(lut_offset<BW, 7>(vw, (S::PT + 2 * j + 1) * BW, lane_lut));
        mma16816(st.O[j], movmatrix_trans(L0), movmatrix_trans(L1), movmatrix_trans(L2),
                 movmatrix_trans(L3), pb0, pb1);
      }
      }   // tile compute
      // ---- refill the stage with this warp's tile of block i + NS --------
      __syncwarp();
      if (!aborted && i + S::NS < nblk) fetch_next(stage, true);
    };

    // The run as segments of one position each: the blocks before a unit's
    // last one are full; its last block holds pos_tail(p) tokens.
    const std::integral_constant<bool, false> full_tile{};
    const std::integral_constant<bool, true> masked_tile{};
    int pos = p_first, blk = blk_first;
    int i = 0;
    while (i < nblk) {
      const int uid = setup_unit(pos);
      const int nbp = pos_blocks(pos), tail = pos_tail(pos);
      const int slot = c - (int)(pos_off(pos) / cold_bpc());
      const int seg = (nbp - blk) < (nblk - i) ? (nbp - blk) : (nblk - i);   // this unit's blocks in the run
      const bool ends_unit = blk + seg == nbp;
      const int n_full = (ends_unit && tail < S::TB) ? seg - 1 : seg;
      const int i_end = i + seg, i_full = i + n_full;
      const int64_t tok_first = (int64_t)(blk - i) * S::TB + tb;   // + 64 i: this warp's first token
      for (; i < i_full; ++i) tile_step(i, full_tile, 16, uid, tok_first + (int64_t)i * S::TB);
      if (i < i_end) {
        const int left = tail - tb;
        tile_step(i, masked_tile, left < 16 ? left : 16, uid, tok_first + (int64_t)i * S::TB);
        ++i;
      }
      flush_partial<D, S::NT, HPL, HMAP>(st, false, inv_levels, G, merge,
                                         a.part + (((size_t)uid * slots + slot) * G) * (D + 2));
      st.reset();
      pos = pos_next(pos);
      blk = 0;
    }
    __syncthreads();
    if (*abort_flag) {
      // A bulk copy did not complete in time: latch the error, give the
      // copies still in flight a bounded chance to land, and leave.
      if (tid == 0) atomicOr(a.status, kStatusTimeout);
      if (lane == 0)             // stage s received copies s, s + NS, ...: wait for its last one
        for (int s = 0; s < S::NS && s < issued; ++s) {
          const int n_s = (issued - s + S::NS - 1) / S::NS;
          mbar_wait_bounded(bar_w + 8 * s, (uint32_t)((n_s - 1) & 1), kDefaultWaitLimitNs);
        }
      return;
    }
  }
  if (c < pl.hot_ctas) {
    // ====== then hot tiles [c * tpc, (c + 1) * tpc): the ring is idle ======
    // units with uniform hot counts, or (ragged) per-row counts with the
    // units' tiles flattened by prefix sums, skipping rows without hot tokens
    const int n_rows = a.units / a.Hkv;
    auto row_tiles = [&](int b) -> int { return (a.rows->n_hot[b] + S::TB - 1) / S::TB; };
    auto unit_tiles = [&](int u) -> int {
      if constexpr (RAGGED) return row_tiles(u / a.Hkv); else return pl.hot_tiles;
    };
    auto unit_hoff = [&](int u) -> int64_t {
      if constexpr (RAGGED) {
        const int b = u / a.Hkv;
        return a.rows->hot_pre[b] + (int64_t)(u % a.Hkv) * row_tiles(b);
      } else {
        return (int64_t)u * pl.hot_tiles;
      }
    };
    auto unit_nhot = [&](int u) -> int {
      if constexpr (RAGGED) return a.rows->n_hot[u / a.Hkv]; else return a.n_hot;
    };
    auto unit_next = [&](int u) -> int {
      if constexpr (RAGGED) {
        if ((u + 1) % a.Hkv != 0) return u + 1;
        int b = (u + 1) / a.Hkv;
        while (b < n_rows && a.rows->n_hot[b] == 0) ++b;
        return b * a.Hkv;
      } else {
        return u + 1;
      }
    };
    const int64_t total = RAGGED ? (int64_t)a.rows->hot_pre[n_rows] : (int64_t)a.units * pl.hot_tiles;
    const int64_t f_lo = (int64_t)c * pl.hot_tpc;
    const int64_t f_hi = f_lo + pl.hot_tpc < total ? f_lo + pl.hot_tpc : total;
    constexpr int CH = D / 8;        // 16-byte chunks per token row
    WarpState<S::NT, 2> sh;          // hot logits use one MMA column per head
    sh.reset();
    uint32_t qh[S::NT][2];
    int unit_cur = -1, slot_cur = 0;
    int unit, tile;
    if constexpr (RAGGED) {
      int lo = 0, hi = n_rows - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.rows->hot_pre[mid] <= f_lo) lo = mid; else hi = mid - 1;
      }
      const int htr = row_tiles(lo);
      const int64_t off = f_lo - a.rows->hot_pre[lo];
      unit = lo * a.Hkv + (int)(off / htr);
      tile = (int)(off % htr);
    } else {
      unit = (int)(f_lo / pl.hot_tiles);
      tile = (int)(f_lo - (int64_t)unit * pl.hot_tiles);
    }
    int ht = unit_tiles(unit);
    for (int64_t f = f_lo; f < f_hi; ++f, ++tile) {
      if (tile == ht) {
        tile = 0;
        unit = unit_next(unit);
        ht = unit_tiles(unit);
      }
      if (unit != unit_cur) {
        if (unit_cur >= 0) {
          flush_partial<D, S::NT, 2, HMAP_PAIR>(sh, true, inv_levels, G, merge,
                                  a.part + (((size_t)unit_cur * slots + slot_cur) * G) * (D + 2));
          sh.reset();
        }
        unit_cur = unit;
        slot_cur = pl.slots_cold + (c - (int)(unit_hoff(unit) / pl.hot_tpc));
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
      const int n_hot_u = unit_nhot(unit);
      // the tile's K rows, then (in the same buffer) its V rows
      auto stage_rows = [&](const __half* src) {
        __syncthreads();
        for (int i = tid; i < S::TB * CH; i += kThreads) {
          const int r = i / CH, cc = i % CH;
          const int slot = tile * S::TB + r;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (slot < n_hot_u)
            v = __ldg(reinterpret_cast<const uint4*>(src + ((size_t)unit * a.W + slot) * D) + cc);
          *reinterpret_cast<uint4*>(ring + r * S::RS + cc * 16) = v;
        }
        __syncthreads();
      };
      const int nvalid = n_hot_u - tile * S::TB < S::TB ? n_hot_u - tile * S::TB : S::TB;
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
      flush_partial<D, S::NT, 2, HMAP_PAIR>(sh, true, inv_levels, G, merge,
                              a.part + (((size_t)unit_cur * slots + slot_cur) * G) * (D + 2));
    }
  }
}

// ---------------------------------------------------------------------------
// Instantiation table of one (D, M).
// ---------------------------------------------------------------------------
typedef void (*AttendFn)(const AttendArgs);

template <int D, int M, int BW, bool SLOT, int HMAP>
AttendFn attend_fn_mode(int mode) {
  if (mode == MODE_GATED) return attend_kernel<D, M, BW, SLOT, HMAP, MODE_GATED>;
  if (mode == MODE_LOGITS) return attend_kernel<D, M, BW, SLOT, HMAP, MODE_LOGITS>;
  if (mode == MODE_RAGGED) return attend_kernel<D, M, BW, SLOT, HMAP, MODE_RAGGED>;
  return attend_kernel<D, M, BW, SLOT, HMAP, MODE_PLAIN>;
}

template <int D, int M, int BW, bool SLOT>
AttendFn attend_fn_bw(int hmap, int mode) {
  if constexpr (SLOT) {
    if (hmap == HMAP_PACK) return attend_fn_mode<D, M, BW, true, HMAP_PACK>(mode);
    return attend_fn_mode<D, M, BW, true, HMAP_SPLIT>(mode);
  } else {
    if (hmap == HMAP_PACK) return attend_fn_mode<D, M, BW, false, HMAP_PACK>(mode);
    return attend_fn_mode<D, M, BW, false, HMAP_PAIR>(mode);
  }
}

// SLOT for b_theta <= 3 (code widths 2..8), HILO for b_theta >= 4 (5..8).
template <int D, int M>
AttendFn attend_fn_dm(int bw, int b_theta, int G, int mode, int* smem) {
  const bool slot = b_theta <= 3;
  const int hmap = G <= 4 ? HMAP_PACK : (slot ? HMAP_SPLIT : HMAP_PAIR);
#define TQ_BW_CASE(B)                                                             \
  case B:                                                                         \
    *smem = AttendShape<D, M, B>::SMEM;                                           \
    if (slot) return attend_fn_bw<D, M, B, true>(hmap, mode);                     \
    if constexpr (B >= 5) return attend_fn_bw<D, M, B, false>(hmap, mode);        \
    return nullptr;
  switch (bw) {
    TQ_BW_CASE(2)
    TQ_BW_CASE(3)
    TQ_BW_CASE(4)
    TQ_BW_CASE(5)
    TQ_BW_CASE(6)
    TQ_BW_CASE(7)
    TQ_BW_CASE(8)
  }
#undef TQ_BW_CASE
  return nullptr;
}

}  // namespace att

// Per-(D, M) pickers, one per instantiation file.
att::AttendFn attend_pick_64_64(int bw, int b_theta, int G, int mode, int* smem);
att::AttendFn attend_pick_64_128(int bw, int b_theta, int G, int mode, int* smem);
att::AttendFn attend_pick_128_64(int bw, int b_theta, int G, int mode, int* smem);
att::AttendFn attend_pick_128_128(int bw, int b_theta, int G, int mode, int* smem);

}  // namespace tq
