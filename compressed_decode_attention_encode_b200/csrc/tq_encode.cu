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
#include "tq_encode_core.cuh"

namespace tq {
namespace {

using namespace enc;

constexpr int kStStageBytes = 64 * 1024;   // largest S^T staged in shared memory

__host__ __device__ constexpr bool st_staged(int d, int m) { return d * m * 4 <= kStStageBytes; }

// Per-block shared memory: [warps][4][D] doubles (the residuals of a warp's
// four keys), per-warp code / sign / scalar staging, then S^T when staged
// (16-byte aligned).
__host__ __device__ constexpr size_t st_offset(int d, int warps) {
  return ((size_t)warps * 4 * d * sizeof(double) + (size_t)warps * (8 * (d / 2) + 4 * 32 + 32) + 15) /
         16 * 16;
}

// encode_small_kernel's shared memory: [2][D] doubles, [2][D/32] doubles,
// [2][D/2] code bytes, 4 sign words, 3 scalars; then S^T (16-byte aligned).
__host__ __device__ constexpr size_t small_st_offset(int d) {
  return ((size_t)2 * d * 8 + (size_t)2 * (d / 32) * 8 + (size_t)d + 16 + 8 + 15) / 16 * 16;
}

// One bulk copy of S^T into shared memory, completed on an mbarrier, and a
// bounded wait for it (a copy that never lands latches kStatusTimeout; the
// decode's merge then writes NaN).
__device__ __forceinline__ void st_bulk_copy(uint32_t bar, void* dst, const void* src, uint32_t bytes) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          (uint32_t)__cvta_generic_to_shared(dst)),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void st_bulk_wait(uint32_t bar, int* status) {
  uint32_t ok = 0;
  uint64_t t0 = 0;
  for (int it = 0;; ++it) {
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0, %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(1000000u)
        : "memory");
    if (ok) return;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (it == 0) t0 = t;
    else if (t - t0 > kDefaultWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// Merges `val` into the 32-bit word at `addr` under `mask` (bits of tokens
// written by this launch); bits of other tokens are kept.
__device__ __forceinline__ void merge_word(uint32_t* addr, uint32_t val, uint32_t mask) {
  if (mask == 0u) return;
  if (mask != 0xffffffffu) val = (*addr & ~mask) | (val & mask);
  *addr = val;
}

// What one launch writes for a unit: n tokens at cold positions cold_start
// .. cold_start + n - 1, the first nA read from ring slots (ring_start + e)
// mod W, the rest from source tokens e - nA.  Uniform over the units, or
// (ragged batch) from the unit's row: an append of n_new tokens, or an
// insert of n_new tokens that evicts max(0, n_hot + n_new - W), the ring's
// oldest first.
struct UnitSpan {
  int64_t cold_start, n;
  int nA, ring_start;
};

__device__ __forceinline__ UnitSpan unit_span(const EncodeArgs& a, int unit) {
  UnitSpan u;
  if (a.rows != nullptr) {
    const RowTable* r = a.rows;
    const int b = unit / a.Hkv;
    u.cold_start = r->n_cold[b];
    if (a.ring_k == nullptr) {
      u.n = r->n_new[b];
      u.nA = 0;
      u.ring_start = 0;
    } else {
      const int e = r->n_hot[b] + r->n_new[b] - a.W;
      u.n = e > 0 ? e : 0;
      u.nA = (int)(u.n < r->n_hot[b] ? u.n : r->n_hot[b]);
      u.ring_start = ((r->ring_pos[b] - r->n_hot[b]) % a.W + a.W) % a.W;
    }
  } else {
    u.cold_start = a.cold_start;
    u.n = (int64_t)a.nA + a.nB;
    u.nA = a.nA;
    u.ring_start = a.ring_start;
  }
  return u;
}

// One warp per group of 4 tokens {2c, 2c+1, 2c+8, 2c+9} of a 16-token tile:
// exactly the tokens whose fragment-major words can share a 32-bit word, so
// no two warps ever write the same word.  D = padded length (power of two).
template <int D>
__global__ void __launch_bounds__(256) encode_kernel(EncodeArgs a) {
  constexpr int P = D / 2;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  extern __shared__ double smem[];
  double* rbuf = smem + warp * 4 * D;        // [4][D] the job's key residuals
  uint8_t* wbase = reinterpret_cast<uint8_t*>(smem + warps * 4 * D) + warp * (8 * P + 4 * 32 + 32);
  uint8_t* kc = wbase;                       // [4][P] key code words
  uint8_t* vc = wbase + 4 * P;               // [4][P] value code words
  uint32_t* kb = reinterpret_cast<uint32_t*>(wbase + 8 * P);   // [4][8] sign words
  uint16_t* sc = reinterpret_cast<uint16_t*>(wbase + 8 * P + 128);  // [4][4] s16_k, rn16, s16_v

  const Layout& L = a.L;
  const int bw = L.bw;
  const int64_t n = (int64_t)a.nA + a.nB;    // (uniform; a ragged launch takes its counts per unit)
  if (a.rows == nullptr && n == 0) return;
  __shared__ double2 atab[kAngleTableEntries];
  angle_tables(1 << L.b_theta, a.atab, atab, threadIdx.x, blockDim.x);
  __syncthreads();
  // S^T in shared memory when it fits: the sign loop then waits on shared
  // memory instead of a chain of L2 round trips (the decode-step eviction
  // encodes one token per unit, so latency is all there is).
  // (m = 64 or 128: S^T in lane order, read by qjl_sketch_lanes)
  const bool lanes = st_staged(D, L.m) && (L.m == 64 || L.m == 128);
  const float* St = a.St;
  float* sst = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(smem) + st_offset(D, warps));
  if (st_staged(D, L.m)) {
    async_copy_g2s(sst, lanes ? a.Stl : a.St, D * L.m * 4);
    async_copy_wait();
    __syncthreads();
    St = sst;
  }
  // uniform: every unit writes the same tile range; ragged: each its own,
  // within groups_max groups
  const int64_t groups = a.rows ? a.groups_max
                                : ((a.cold_start + n - 1) / kTokensPerTile - a.cold_start / kTokensPerTile + 1) * 4;
  const int64_t jobs = (int64_t)a.units * groups;

  for (int64_t job = (int64_t)blockIdx.x * warps + warp; job < jobs;
       job += (int64_t)gridDim.x * warps) {
    const int unit = (int)(job / groups);
    const int64_t g = job % groups;
    const UnitSpan us = unit_span(a, unit);
    if (us.n == 0) continue;
    const int64_t t_first = us.cold_start / kTokensPerTile;
    if (g >= ((us.cold_start + us.n - 1) / kTokensPerTile - t_first + 1) * 4) continue;
    const int64_t tile = t_first + g / 4;
    const int c = (int)(g % 4);
    bool inr[4];
    int64_t seq[4];
    bool any = false;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = 2 * c + (s & 1) + 8 * (s >> 1);
      const int64_t t = tile * kTokensPerTile + r;
      seq[s] = t - us.cold_start;
      inr[s] = seq[s] >= 0 && seq[s] < us.n;
      any |= inr[s];
    }
    if (!any) continue;
    const unsigned inm = (unsigned)inr[0] | ((unsigned)inr[1] << 1) | ((unsigned)inr[2] << 2) |
                         ((unsigned)inr[3] << 3);   // (bit s: token s is written)
    for (int s = 0; s < 4; ++s) {
      if (!inr[s]) continue;
      const int64_t e = seq[s];
      const __half* ksrc;
      const __half* vsrc;
      if (e < us.nA) {
        const int slot = (int)((us.ring_start + e) % a.W);
        ksrc = a.ring_k + ((int64_t)unit * a.W + slot) * D;
        vsrc = a.ring_v + ((int64_t)unit * a.W + slot) * D;
      } else {
        ksrc = a.src_k + ((int64_t)unit * a.src_tokens + (e - us.nA)) * D;
        vsrc = a.src_v + ((int64_t)unit * a.src_tokens + (e - us.nA)) * D;
      }
      encode_kv_pair<D>(a.L, a.signs, atab, a.inv_sqrt_d, a.status, ksrc, vsrc, rbuf + s * D, kc + s * P,
                        vc + s * P, sc + s * 4, sc + s * 4 + 1, sc + s * 4 + 2);
    }
    // the four keys' sign words in one pass over S^T (lane order when staged
    // for m = 64 or 128)
    if (lanes && L.m == 128) qjl_sketch_lanes<D, 4, 4>(sst, rbuf, inr, kb, 8);
    else if (lanes) qjl_sketch_lanes<D, 4, 2>(sst, rbuf, inr, kb, 8);
    else if (L.m <= 128) qjl_sketch_block<D, 4, 4>(L.m, St, rbuf, inr, kb, 8);
    else qjl_sketch_block<D, 4, 8>(L.m, St, rbuf, inr, kb, 8);
    __syncwarp();

    uint8_t* tb = a.cold + ((int64_t)unit * L.blocks_per_unit + tile / kTilesPerBlock) * L.block_bytes +
                  (tile % kTilesPerBlock) * L.tile_bytes;
    // ---- the job's fields into the fragment-major words ------------------
    // Lane chunk ch = 4 e + tig (tile lane 4 (2c + e) + tig) holds codes
    // q = h PT + k (pair tig PT + k of token e + 2h) at chunk bit q bw.
    // Codes: lane (kv, ch, h) packs its PT codes into whole words with a
    // 64-bit shift register; when PT bw is not a multiple of 32 the two
    // halves share a word, which the h = 0 lane completes with its
    // neighbour's part.  Only bits of tokens this launch writes are merged.
    {
      constexpr int PT = P / 4;
      const int kv = lane >> 4, ch = (lane >> 1) & 7, h = lane & 1;
      const int e = ch >> 2, tig = ch & 3, sl = e + 2 * h;
      const int l = 4 * (2 * c + e) + tig;
      const uint32_t* src = reinterpret_cast<const uint32_t*>((kv ? vc : kc) + sl * P + tig * PT);
      uint8_t* plane = tb + (kv ? L.off_vc : L.off_kc);
      const int nw = kv ? L.vwt : L.kwt;
      const bool live = (inm >> sl) & 1u;
      const uint32_t cm = live ? (1u << bw) - 1u : 0u;
      const bool shared = ((PT * bw) & 31) != 0;
      const int bit0 = h * PT * bw;
      int w = bit0 >> 5, nb = bit0 & 31;
      uint64_t acc = 0u, am = 0u;
      uint32_t hv = 0u, hm = 0u;         // h = 1: its part of the shared word
      bool first = true;
#pragma unroll
      for (int k4 = 0; k4 < PT / 4; ++k4) {
        const uint32_t cw = live ? src[k4] : 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc |= (uint64_t)((cw >> (8 * k)) & 0xffu) << nb;
          am |= (uint64_t)cm << nb;
          nb += bw;
          if (nb >= 32) {
            if (h == 1 && first && shared) {
              hv = (uint32_t)acc;
              hm = (uint32_t)am;
            } else {
              merge_word(reinterpret_cast<uint32_t*>(plane + lane_word_offset(w, l, nw)), (uint32_t)acc,
                         (uint32_t)am);
            }
            first = false;
            acc >>= 32;
            am >>= 32;
            nb -= 32;
            ++w;
          }
        }
      }
      const uint32_t ov = __shfl_down_sync(kFull, hv, 1), om = __shfl_down_sync(kFull, hm, 1);
      if (nb > 0)   // h = 0: the shared word; h = 1: the chunk's last, partial word
        merge_word(reinterpret_cast<uint32_t*>(plane + lane_word_offset(w, l, nw)),
                   (uint32_t)acc | (h == 0 ? ov : 0u), (uint32_t)am | (h == 0 ? om : 0u));
    }
    // Signs (m = 64 or 128): local sign j of token half h sits at chunk bit
    // sign_chunk_bit(j, h, m); lane (ch, h) < 16 permutes its token's m/4
    // signs of this chunk with compile-time positions (m = 64: both halves
    // share the word, combined by shuffle).
    {
      const int ch = (lane >> 1) & 7, h = lane & 1;
      const int e = ch >> 2, tig = ch & 3, sl = e + 2 * h;
      const int l = 4 * (2 * c + e) + tig;
      const bool live = lane < 16 && ((inm >> sl) & 1u);
      const int qb = L.m / 4;
      const uint32_t kw = live ? kb[sl * 8 + ((tig * qb) >> 5)] >> ((tig * qb) & 31) : 0u;
      uint32_t pv = 0u, pm = 0u;
      if (L.m == 128) {
#pragma unroll
        for (int j = 0; j < 32; ++j) pv |= ((kw >> j) & 1u) << sign_chunk_bit(j, 0, 128);
        pm = live ? 0xffffffffu : 0u;
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) pv |= ((kw >> j) & 1u) << sign_chunk_bit(j, 0, 64);
        pv <<= 4 * h;
        pm = live ? 0x0f0f0f0fu << (4 * h) : 0u;
        pv |= __shfl_xor_sync(kFull, pv, 1);
        pm |= __shfl_xor_sync(kFull, pm, 1);
      }
      if (lane < 16 && (L.m == 128 || h == 0))
        merge_word(reinterpret_cast<uint32_t*>(tb + L.off_ks + lane_word_offset(L.m == 128 ? h : 0, l, L.sw)),
                   pv, pm);
    }
    // scalars
    if (lane < 4 && ((inm >> lane) & 1u)) {
      const int s = lane;
      const int e = s & 1, h = s >> 1, gid = 2 * c + e;
      uint16_t* ks = reinterpret_cast<uint16_t*>(tb + L.off_ksc);
      uint16_t* vs = reinterpret_cast<uint16_t*>(tb + L.off_vsc);
      ks[gid * 4 + h] = sc[s * 4];
      ks[gid * 4 + 2 + h] = sc[s * 4 + 1];
      vs[gid * 2 + h] = sc[s * 4 + 2];
    }
    __syncwarp();
  }
}

// Latency path for a few tokens per unit (the decode-step eviction): one
// CTA per (unit, token); threads [0, D) encode the key with one element per
// thread, threads [D, 2D) the value.  The float64 operations are those of
// encode_vector_any (the polar and residual steps run on one thread per
// pair, in parallel instead of PL pairs in turn per lane), so the codes
// match the float64 definition the same way.  The token's fields are merged
// into the fragment-major words with atomicAnd / atomicOr: CTAs writing
// other tokens of the same words never lose each other's bits.
template <int D>
__global__ void __launch_bounds__(2 * D) encode_small_kernel(EncodeArgs a) {
  constexpr int P = D / 2;
  constexpr int NW = D / 32;                 // warps per team
  const Layout& L = a.L;
  // (a few tokens per unit: 32-bit index arithmetic)
  const int n = a.promo ? kPromoMax + a.n_new : a.rows ? a.n_max : (int)(a.nA + a.nB);
  const int unit = (int)blockIdx.x / n;
  const int e = (int)blockIdx.x % n;
  const int tid = threadIdx.x, team = tid / D, el = tid % D;
  const int lane = tid & 31, wt = el >> 5;
  // A following launch that opted in (the decode step's q-prep, which does
  // not read what this kernel writes) may start now.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ double sm[];
  double* xb = sm + team * D;                                  // [2][D] exchange / residual
  double* red = sm + 2 * D;                                    // [2][NW] reductions
  uint8_t* codes = reinterpret_cast<uint8_t*>(red + 2 * NW);   // [2][P] key / value codes
  uint32_t* bits = reinterpret_cast<uint32_t*>(codes + 2 * P); // [4] key sign words
  uint16_t* sc = reinterpret_cast<uint16_t*>(bits + 4);        // s16_k, rn16, s16_v
  float* sst = reinterpret_cast<float*>(sm) + small_st_offset(D) / 4;   // S^T [D][m]
  __shared__ uint64_t st_bar;
  __shared__ double2 atab[kAngleTableEntries];
  const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&st_bar);
  // S^T lands while the rotation and polar steps run (one bulk copy); the
  // angle tables are published by the rotation's first block barrier
  if (tid == 0) st_bulk_copy(bar, sst, a.St, (uint32_t)(D * L.m * 4));
  angle_tables(1 << L.b_theta, a.atab, atab, tid, blockDim.x);
  // Launched as a programmatic dependent of the kernel before it: S^T (set
  // at cache creation) may be fetched early, the inputs only once that
  // kernel has finished.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const __half* src;
  int64_t dest = a.cold_start + e;           // cold position written
  const __half* nsrc = nullptr;              // the slot's new occupant (write_new)
  if (a.promo) {
    // insert e of this unit: its promoted tokens first, then the new ones
    const PromoUnitState* st = a.promo + unit;
    const int k = st->n_pend;
    if (e >= k + a.n_new) {                  // (the whole CTA) nothing to insert
      if (tid == 0) st_bulk_wait(bar, a.status);
      return;
    }
    const int slot = (int)((st->ring_pos + e) % a.W);
    src = (team ? a.ring_v : a.ring_k) + ((int64_t)unit * a.W + slot) * D;
    if (e < k) {
      dest = st->pend_idx[e];
      nsrc = (team ? a.promo_v : a.promo_k) + ((int64_t)unit * kPromoMax + e) * D;
    } else {
      dest = a.cold_start + (e - k);
      nsrc = (team ? a.src_v : a.src_k) + ((int64_t)unit * a.src_tokens + (e - k)) * D;
    }
  } else {
    const UnitSpan us = unit_span(a, unit);
    if (e >= us.n) {                         // (the whole CTA) nothing for this unit
      if (tid == 0) st_bulk_wait(bar, a.status);
      return;
    }
    dest = us.cold_start + e;
    if (e < us.nA) {
      const int slot = (int)((us.ring_start + e) % a.W);
      src = (team ? a.ring_v : a.ring_k) + ((int64_t)unit * a.W + slot) * D;
      if (a.write_new) nsrc = (team ? a.src_v : a.src_k) + ((int64_t)unit * a.src_tokens + e) * D;
    } else {
      src = (team ? a.src_v : a.src_k) + ((int64_t)unit * a.src_tokens + (e - us.nA)) * D;
    }
  }
  // ---- rotation: y = H (D x) / sqrt(d) ----------------------------------
  const __half xin = src[el];
  if (nsrc) const_cast<__half*>(src)[el] = nsrc[el];   // the slot just read takes its new occupant
  double x = __dmul_rn((double)__half2float(xin), a.signs[el]);
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    double o;
    if (h < 32) {
      o = __shfl_xor_sync(kFull, x, h);
    } else {
      xb[el] = x;
      __syncthreads();
      o = xb[el ^ h];
      __syncthreads();
    }
    x = (el & h) ? __dsub_rn(o, x) : __dadd_rn(x, o);
  }
  x = __dmul_rn(x, a.inv_sqrt_d);

  // ---- polar (even threads own pair el / 2) -------------------------------
  const double y1 = __shfl_xor_sync(kFull, x, 1);
  const bool ev = !(el & 1);
  const int nt = 1 << L.b_theta;
  double rho = 0.0;
  int ct = 0;
  if (ev) {
    rho = __dsqrt_rn(__dadd_rn(__dmul_rn(x, x), __dmul_rn(y1, y1)));
    ct = angle_code(x, y1, nt, atab);
  }
  double mr = rho;
#pragma unroll
  for (int o = 16; o; o >>= 1) mr = fmax(mr, __shfl_xor_sync(kFull, mr, o));
  if (lane == 0) red[team * NW + wt] = mr;
  __syncthreads();
  double smax = red[team * NW];
#pragma unroll
  for (int w = 1; w < NW; ++w) smax = fmax(smax, red[team * NW + w]);
  uint16_t s16b = f64_to_f16_bits(smax);
  if ((s16b & 0x7c00u) == 0x7c00u) {
    if (el == 0) atomicOr(a.status, kStatusRange);
    s16b = 0;
  }
  const double s16 = f16_bits_to_f64(s16b);
  const bool zero = (s16 == 0.0);
  const int Lr = (1 << L.b_r) - 1;
  int cr = 0;
  if (ev) {
    const double tr = __dmul_rn(__ddiv_rn(rho, zero ? 1.0 : s16), (double)Lr);
    const int c = (int)rint(tr);
    cr = c < 0 ? 0 : (c > Lr ? Lr : c);
    if (zero) { cr = 0; ct = 0; }
    codes[team * P + el / 2] = (uint8_t)((cr << L.b_theta) | ct);
  }
  if (el == 0) sc[team ? 2 : 0] = s16b;

  // ---- keys: residual, its norm and the QJL signs --------------------------
  double ss = 0.0;
  if (team == 0 && ev) {
    const double rh = __ddiv_rn(__dmul_rn((double)cr, s16), (double)Lr);
    const double2 csn = atab[angle_cs_offset(nt) + ct];     // cos, sin of c_theta 2 pi / nt
    const double r0 = __dsub_rn(x, __dmul_rn(rh, csn.x));
    const double r1 = __dsub_rn(y1, __dmul_rn(rh, csn.y));
    xb[el] = r0;
    xb[el + 1] = r1;
    ss = __dadd_rn(__dmul_rn(r0, r0), __dmul_rn(r1, r1));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
  st_bulk_wait(bar, a.status);
  __syncthreads();            // residual complete, S^T staged, reduction slots free
  if (team == 0) {
    if (lane == 0) red[wt] = ss;
  }
  __syncthreads();
  if (team == 0 && el == 0) {
    double tot = red[0];
    for (int w = 1; w < NW; ++w) tot = __dadd_rn(tot, red[w]);
    const uint16_t rnb = f64_to_f16_bits(__dsqrt_rn(tot));
    if ((rnb & 0x7c00u) == 0x7c00u) atomicOr(a.status, kStatusRange);
    sc[1] = rnb;
  }
  // (S r)_i: team t sums j in [t D/2, (t + 1) D/2) as four interleaved
  // partial sums; team 1 hands its half to team 0 through its (now free)
  // exchange buffer.  A sign can differ from another summation order only
  // within float64 rounding of zero.
  const double* rres = sm;                   // the key residual (team 0's buffer)
  double* pbuf = sm + D;
  for (int i0 = 0; i0 < L.m; i0 += D) {
    const int i = i0 + el;
    double part = 0.0;
    if (i < L.m) {
      double p4[4] = {0.0, 0.0, 0.0, 0.0};
      const int j0 = team * (D / 2);
#pragma unroll 4
      for (int j = j0; j < j0 + D / 2; j += 4) {
#pragma unroll
        for (int t = 0; t < 4; ++t) p4[t] = fma((double)sst[(j + t) * L.m + i], rres[j + t], p4[t]);
      }
      part = __dadd_rn(__dadd_rn(p4[0], p4[1]), __dadd_rn(p4[2], p4[3]));
    }
    if (team == 1) pbuf[el] = part;
    __syncthreads();
    if (team == 0) {
      const double acc = __dadd_rn(part, pbuf[el]);
      const unsigned word = __ballot_sync(kFull, i < L.m && acc >= 0.0);
      if (lane == 0 && i < L.m) bits[i >> 5] = word;
    }
    __syncthreads();
  }

  // ---- merge the token's fields into its tile ------------------------------
  const int64_t tok = dest;
  const int64_t tile = tok / kTokensPerTile;
  const int r = (int)(tok % kTokensPerTile), gid = r % 8, h = r / 8;
  uint8_t* tb = a.cold + ((int64_t)unit * L.blocks_per_unit + tile / kTilesPerBlock) * L.block_bytes +
                (tile % kTilesPerBlock) * L.tile_bytes;
  auto merge_atomic = [](uint8_t* addr, uint32_t val, uint32_t mask) {
    if (mask == 0u) return;
    uint32_t* w = reinterpret_cast<uint32_t*>(addr);
    atomicAnd(w, ~mask);
    atomicOr(w, val & mask);
  };
  const int bw = L.bw;
  constexpr int PT = P / 4;                  // pairs per lane group and token
  const uint32_t cm = (1u << bw) - 1u;
  const int nwarps = blockDim.x >> 5, warp = tid >> 5;
  // One warp per (plane, lane group tg) and word: lane k holds this token's
  // code k (pair tg * PT + k, at bit (h PT + k) bw of the group's stream) or
  // sign bit k, and the word's bits and mask come from two OR-reductions.
  // Jobs 0-3: key codes, 4-7: value codes, 8-11: sign words.
  for (int job = warp; job < 12; job += nwarps) {
    const int tg = job & 3;
    if (job < 8) {
      const bool vplane = job >= 4;
      const int nw = vplane ? L.vwt : L.kwt;
      uint8_t* plane = tb + (vplane ? L.off_vc : L.off_kc);
      const uint32_t c = lane < PT ? codes[(vplane ? P : 0) + tg * PT + lane] : 0u;
      const int bit0 = (h * PT + lane) * bw;
      const int w_lo = (h * PT * bw) >> 5, w_hi = ((h + 1) * PT * bw - 1) >> 5;
      for (int w = w_lo; w <= w_hi; ++w) {
        uint32_t v = 0u, mk = 0u;
        const int b = bit0 - 32 * w;
        if (lane < PT && b > -bw && b < 32) {
          v = b >= 0 ? c << b : c >> -b;
          mk = b >= 0 ? cm << b : cm >> -b;
        }
        v = __reduce_or_sync(kFull, v);
        mk = __reduce_or_sync(kFull, mk);
        if (lane == 0) merge_atomic(plane + lane_word_offset(w, 4 * gid + tg, nw), v, mk);
      }
    } else {
      // sign j of this token and lane group: canonical index tg * m/4 + j,
      // chunk bit sign_chunk_bit(j, h, m)
      const int qb = L.m / 4;
      uint32_t bitv = 0u;
      int pos = -1;
      if (lane < qb) {
        const int i = tg * qb + lane;
        bitv = (bits[i >> 5] >> (i & 31)) & 1u;
        pos = sign_chunk_bit(lane, h, L.m);
      }
      for (int w = 0; w < L.sw; ++w) {
        const bool mine = pos >= 32 * w && pos < 32 * w + 32;
        const uint32_t v = __reduce_or_sync(kFull, mine ? bitv << (pos - 32 * w) : 0u);
        const uint32_t mk = __reduce_or_sync(kFull, mine ? 1u << (pos - 32 * w) : 0u);
        if (lane == 0) merge_atomic(tb + L.off_ks + lane_word_offset(w, 4 * gid + tg, L.sw), v, mk);
      }
    }
  }
  if (tid == 0) {
    uint16_t* ks = reinterpret_cast<uint16_t*>(tb + L.off_ksc);
    uint16_t* vs = reinterpret_cast<uint16_t*>(tb + L.off_vsc);
    ks[gid * 4 + h] = sc[0];
    ks[gid * 4 + 2 + h] = sc[1];
    vs[gid * 2 + h] = sc[2];
  }
}

__global__ void ring_write_kernel(__half* ring_k, __half* ring_v, const __half* k_new,
                                  const __half* v_new, int units, int W, int d, int n,
                                  int first, int ring_pos, const RowTable* rows, int Hkv) {
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
    int rp = ring_pos;
    if (rows != nullptr) {          // ragged: row b writes its tokens [max(0, n_b - W), n_b)
      const int b = unit / Hkv, nb = rows->n_new[b];
      if (i >= nb || i < nb - W) continue;
      rp = rows->ring_pos[b];
    }
    const int slot = (int)(((int64_t)rp + i) % W);
    const uint4* s = reinterpret_cast<const uint4*>((is_k ? k_new : v_new) + ((int64_t)unit * n + i) * d) + c;
    uint4* dst = reinterpret_cast<uint4*>((is_k ? ring_k : ring_v) + ((int64_t)unit * W + slot) * d) + c;
    *dst = *s;
  }
}

template <int D>
cudaError_t launch_encode_d(const EncodeArgs& a, cudaStream_t s) {
  const int warps = 8;
  const int64_t n = a.promo ? (int64_t)(kPromoMax + a.n_new)
                  : a.rows ? (int64_t)a.n_max : (int64_t)a.nA + a.nB;
  if (n == 0) return cudaSuccess;
  if (D <= 128 && (n <= kSmallEncodeTokens || a.promo)) {
    const size_t smem = small_st_offset(D) + (size_t)D * a.L.m * sizeof(float);
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(encode_small_kernel<D>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.units * n));
    cfg.blockDim = dim3(2 * D);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_small_kernel<D>, a);
  }
  const int64_t jobs = a.rows ? (int64_t)a.units * a.groups_max
                               : (int64_t)a.units * 4 *
                                     ((a.cold_start + n - 1) / kTokensPerTile - a.cold_start / kTokensPerTile + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (jobs + warps - 1) / warps;
  const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
  size_t smem = st_offset(D, warps);
  if (st_staged(D, a.L.m)) smem += (size_t)D * a.L.m * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(encode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
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
                              int ring_pos, cudaStream_t s, const RowTable* rows, int Hkv) {
  const int64_t total = 2 * (int64_t)units * (n - first) * (d / 8);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int grid = (int)(want < 4096 ? want : 4096);
  ring_write_kernel<<<grid, threads, 0, s>>>(ring_k, ring_v, k_new, v_new, units, W, d, n, first,
                                             ring_pos, rows, Hkv);
  return cudaGetLastError();
}

}  // namespace tq
