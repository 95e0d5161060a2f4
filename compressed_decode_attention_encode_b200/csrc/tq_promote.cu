// Attention-weighted promotion with sticky counters ("Monarch v3 ...",
// section "Cómo funciona", item "Promoción Ponderada por Atención": cold
// tokens that draw much attention return to the hot region, and a
// persistence count keeps them from bouncing; the page's benchmark runs it
// with a promotion threshold of 0.15 and a sticky count of 3).
//
// Per decode call (after the merge):
//   promo_mass_kernel  one CTA per (row, kv head) unit.  A cold token's mass
//                      is the mean over the unit's query heads of its final
//                      softmax weight 2^(l - M) / L (its log2-domain logits
//                      from the attention kernel, each head's M and L from
//                      the merge).  Tokens with mass >= threshold are hits;
//                      with threshold >= 1/8 there are at most 8 per unit
//                      (the cold masses sum to at most 1).  A hit's count is
//                      its previous count + 1 (0 if it missed last step);
//                      at the sticky count it is promoted and its count
//                      cleared.  Promotions are kept only while the hot
//                      window is full.
// Per eviction that follows (before the eviction encode):
//   promo_dequant_kernel  the promoted tokens' K and V, R^T (s16/(2^b_r-1)
//                      c_r (cos, sin)), in float64 rounded to fp16.
// and after it:
//   promo_ring_kernel  each unit's ring position advances by its inserts.
#include <cmath>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr double kTwoPi = 6.283185307179586476925286766559;   // rounds to 2 * fp64(pi)
constexpr int kMassThreads = 256;

__global__ void __launch_bounds__(kMassThreads) promo_mass_kernel(const PromoArgs a) {
  __shared__ int hits[2 * kPromoMax];
  __shared__ int n_hits;
  __shared__ float mref[8], linv[8];
  const int u = blockIdx.x;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  const int head0 = b * a.Hq + kvh * a.G;
  if (threadIdx.x == 0) n_hits = 0;
  if (threadIdx.x < a.G) {
    const float* ml = a.ml + 2 * (size_t)(head0 + threadIdx.x);
    const bool any = ml[0] > -INFINITY && ml[1] > 0.f;   // the head attended something
    mref[threadIdx.x] = any ? ml[0] : 0.f;
    linv[threadIdx.x] = any ? 1.f / ml[1] : 0.f;
  }
  __syncthreads();
  const float inv_g = 1.f / (float)a.G;
  const float* lg = a.logits + (size_t)u * a.capacity * a.G;
  for (int64_t t = threadIdx.x; t < a.n_cold; t += blockDim.x) {
    float mass = 0.f;
    for (int g = 0; g < a.G; ++g) mass += exp2f(lg[t * a.G + g] - mref[g]) * linv[g];
    mass *= inv_g;
    if (mass >= a.threshold) {
      const int k = atomicAdd(&n_hits, 1);
      if (k < 2 * kPromoMax) hits[k] = (int)t;
    }
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const int n = n_hits < kPromoMax ? n_hits : kPromoMax;   // never more for threshold >= 1/8
  for (int i = 1; i < n; ++i)                         // ascending cold positions
    for (int j = i; j > 0 && hits[j - 1] > hits[j]; --j) {
      const int x = hits[j]; hits[j] = hits[j - 1]; hits[j - 1] = x;
    }
  PromoUnitState* st = a.state + u;
  int new_idx[kPromoMax], new_cnt[kPromoMax], nn = 0, np = 0;
  int pend[kPromoMax];
  for (int i = 0; i < n; ++i) {
    int c = 1;
    for (int j = 0; j < st->n_cnt; ++j)
      if (st->cnt_idx[j] == hits[i]) c = st->cnt_val[j] + 1;
    if (c >= a.sticky) {
      if (a.ring_full) pend[np++] = hits[i];       // promoted (count cleared)
    } else {
      new_idx[nn] = hits[i];
      new_cnt[nn++] = c;
    }
  }
  for (int i = 0; i < kPromoMax; ++i) {
    st->cnt_idx[i] = i < nn ? new_idx[i] : -1;
    st->cnt_val[i] = i < nn ? new_cnt[i] : 0;
    st->pend_idx[i] = i < np ? pend[i] : -1;
  }
  st->n_cnt = nn;
  st->n_pend = np;
}

// One CTA per (unit, pending slot j); threads [0, D) the key, [D, 2D) the
// value, one element each.  The arithmetic follows the float64 definition:
// y_2p = (s16 / L) (c_r cos th), y_2p+1 = (s16 / L) (c_r sin th) with
// th = (c_th 2 pi) / 2^b_th, then the Hadamard butterflies, 1/sqrt(d) and
// the rotation signs, then fp16 rounding (to nearest even).
template <int D>
__global__ void __launch_bounds__(2 * D) promo_dequant_kernel(const PromoArgs a) {
  __shared__ double xb[2][D];
  const int u = blockIdx.x / kPromoMax, j = blockIdx.x % kPromoMax;
  const PromoUnitState* st = a.state + u;
  if (j >= st->n_pend) return;
  const int team = threadIdx.x / D, el = threadIdx.x % D;
  const Layout& L = a.L;
  const int64_t tok = st->pend_idx[j];
  const uint8_t* tile = a.cold + ((size_t)u * L.blocks_per_unit + tok / kTokensPerBlock) * L.block_bytes +
                        ((tok % kTokensPerBlock) / kTokensPerTile) * L.tile_bytes;
  const int r = (int)(tok % kTokensPerTile), gid = r % 8, h = r / 8;
  // the pair of element el: lane (gid, tig) of the K-layout code stream
  const int p = el / 2, tig = p / L.pt, k = p % L.pt;
  const uint8_t* plane = tile + (team ? L.off_vc : L.off_kc);
  const int nw = team ? L.vwt : L.kwt;
  const int bit = (h * L.pt + k) * L.bw, wi = bit >> 5, bi = bit & 31;
  uint64_t w = *reinterpret_cast<const uint32_t*>(plane + lane_word_offset(wi, 4 * gid + tig, nw));
  if (bi + L.bw > 32 && wi + 1 < nw)
    w |= (uint64_t)*reinterpret_cast<const uint32_t*>(plane + lane_word_offset(wi + 1, 4 * gid + tig, nw)) << 32;
  const int code = (int)((w >> bi) & ((1u << L.bw) - 1u));
  const int cr = code >> L.b_theta, ct = code & ((1 << L.b_theta) - 1);
  const uint16_t s16b = team ? reinterpret_cast<const uint16_t*>(tile + L.off_vsc)[gid * 2 + h]
                             : reinterpret_cast<const uint16_t*>(tile + L.off_ksc)[gid * 4 + h];
  const double s16 = (double)__half2float(__ushort_as_half(s16b));
  const double th = __ddiv_rn(__dmul_rn((double)ct, kTwoPi), (double)(1 << L.b_theta));
  double sn, cs;
  sincos(th, &sn, &cs);
  const double scale = __ddiv_rn(s16, (double)((1 << L.b_r) - 1));
  double x = __dmul_rn(scale, __dmul_rn((double)cr, (el & 1) ? sn : cs));
  // unnormalised Sylvester Hadamard transform, stages h = 1, 2, 4, ...
  for (int hh = 1; hh < D; hh <<= 1) {
    xb[team][el] = x;
    __syncthreads();
    const double o = xb[team][el ^ hh];
    __syncthreads();
    x = (el & hh) ? __dsub_rn(o, x) : __dadd_rn(x, o);
  }
  x = __dmul_rn(__dmul_rn(x, a.inv_sqrt_d), a.signs[el]);
  __half* dst = (team ? a.promo_v : a.promo_k) + ((size_t)u * kPromoMax + j) * D;
  uint16_t hbits;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(hbits) : "d"(x));
  dst[el] = __ushort_as_half(hbits);
}

// The ring positions after an eviction: set to `set_to` (>= 0, every unit)
// or advanced by each unit's inserts (pending promotions + n new tokens);
// the pending lists are consumed.
__global__ void promo_ring_kernel(PromoUnitState* state, int units, int W, int n_new, int set_to) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= units) return;
  PromoUnitState* st = state + u;
  if (set_to >= 0) {
    st->ring_pos = set_to;
  } else {
    st->ring_pos = (st->ring_pos + st->n_pend + n_new) % W;
  }
  st->n_pend = 0;
  for (int i = 0; i < kPromoMax; ++i) st->pend_idx[i] = -1;
}

}  // namespace

cudaError_t launch_promo_mass(const PromoArgs& a, cudaStream_t s) {
  promo_mass_kernel<<<a.units, kMassThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_promo_dequant(const PromoArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)(a.units * kPromoMax);
  switch (a.L.d) {
    case 64: promo_dequant_kernel<64><<<grid, 128, 0, s>>>(a); break;
    case 128: promo_dequant_kernel<128><<<grid, 256, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_promo_ring(PromoUnitState* state, int units, int W, int n_new, int set_to,
                              cudaStream_t s) {
  promo_ring_kernel<<<(units + 127) / 128, 128, 0, s>>>(state, units, W, n_new, set_to);
  return cudaGetLastError();
}

}  // namespace tq
