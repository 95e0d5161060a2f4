// Internal declarations shared by the library's CUDA translation units.
// Layout of the packed cold store, kernel argument blocks and launchers.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/tq.h"

namespace tq {

// Tokens per cold block (one bulk copy) and per tile (one warp's MMA rows).
constexpr int kTokensPerBlock = 64;
constexpr int kTokensPerTile = 16;
constexpr int kTilesPerBlock = kTokensPerBlock / kTokensPerTile;

// Device status word bits (latched, cleared by tq_get_status).
constexpr int kStatusRange = 1;
constexpr int kStatusTimeout = 2;
constexpr int kStatusLayout = 4;    // a kernel found shared memory where its layout does not fit
// Latched errors after which an attention launch wrote no partials: while
// one is latched, the merge writes NaN rather than stale partials.
constexpr int kStatusNoPartials = kStatusTimeout | kStatusLayout;

// Default limit of the attention kernel's bounded mbarrier waits.
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

// Cold-store layout.  Per (row, kv head): 64-token blocks of 4 tiles.  A
// tile (16 tokens) is laid out fragment-major for the decode warp that
// reads it: lane l = 4*gid + tig owns
//   K codes : tokens gid and gid+8, pairs [tig*PT, tig*PT + PT), PT = d/8
//             (code k of token half h at bit (h*PT + k)*bw of the lane chunk)
//   K signs : tokens gid and gid+8, sign bits [tig*m/4, (tig+1)*m/4); local
//             sign j = 8 s + 4 hf + e (e < 4) of token half h sits at bit
//             8 e + 2 s + hf of word h (m = 128) or at bit 8 e + 4 h + 2 s +
//             hf of word 0 (m = 64): a shift by 2 s + hf (+ 4 h) and a mask
//             0x01010101 give the 0/1 bytes of one int8 MMA operand
//   V codes : as the K codes (tokens gid and gid+8, pairs [tig*PT,
//             tig*PT + PT)): a lane's looked-up pair is one row of an 8x8
//             [token x dim] fragment, which movmatrix turns into the
//             [dim x token] operand of the P V product
// Per-lane word streams are stored "2-word-major": words 2g, 2g+1 of every
// lane sit together (8 bytes per lane) so a warp reads them with one
// conflict-free 64-bit load.  Per-token scalars are grouped by gid:
//   K scalars [gid][s16(gid), s16(gid+8), rn16(gid), rn16(gid+8)]
//   V scalars [gid][s16(gid), s16(gid+8)]
// Planes inside a tile: K codes | K signs | K scalars (64 B) | V codes |
// V scalars (32 B); every plane size is a multiple of 16 bytes.
struct Layout {
  int d;            // head_dim (power of two)
  int pairs;        // d / 2
  int b_r, b_theta, bw;
  int m;            // QJL bits
  int kc_bytes;     // canonical packed code bytes per vector: pairs * bw / 8
  int sg_bytes;     // m / 8
  int pt;           // pairs per lane (per token) in the K and V fragments
  int kwt, sw, vwt; // 32-bit words per lane: K codes, K signs, V codes
  int off_kc, off_ks, off_ksc, off_vc, off_vsc;   // plane offsets inside a tile
  int tile_bytes;
  int block_bytes;
  int64_t blocks_per_unit;  // ceil(cold_capacity / 64)
};

__host__ __device__ inline int words_for_bits(int bits) { return (bits + 31) / 32; }

// Byte offset of word w (of nw) of lane l in a 2-word-major plane.
__host__ __device__ inline int lane_word_offset(int w, int l, int nw) {
  const int width = ((w | 1) < nw) ? 8 : 4;
  return (w >> 1) * 256 + l * width + (w & 1) * 4;
}

// Bit of the lane's sign chunk (words concatenated) holding local sign j
// (0 <= j < m/4) of token half h.
__host__ __device__ inline int sign_chunk_bit(int j, int h, int m) {
  const int e = j & 3, hf = (j >> 2) & 1, s = j >> 3;
  return m == 128 ? 32 * h + 8 * e + 2 * s + hf : 8 * e + 4 * h + 2 * s + hf;
}

// Angle tables of the encoders (see angle_tables): at most 2^7 angle codes.
constexpr int kMaxAngleCodes = 128;
constexpr int kAngleTableEntries = kMaxAngleCodes / 4 + kMaxAngleCodes;

__host__ __device__ constexpr int angle_cs_offset(int nt) { return nt >= 4 ? nt / 4 : 1; }

// Host: the (cos, sin) entries for nt angle codes into out[2 e], out[2 e + 1]
// (entries: the half-sector rotation, the first quadrant's inner sector
// boundaries, then the nt code directions c 2 pi / nt).
inline void angle_table_host(int nt, double* out) {
  const double two_pi = 6.283185307179586476925286766559;
  const int nb = angle_cs_offset(nt);
  for (int e = 0; e < nb + nt; ++e) {
    const double a = e == 0 ? two_pi / 2.0 / (double)nt
                   : e < nb ? two_pi * (double)e / (double)nt
                            : (double)(e - nb) * two_pi / (double)nt;
    out[2 * e] = std::cos(a);
    out[2 * e + 1] = std::sin(a);
  }
}

__host__ __device__ inline Layout layout_of(int d, int b_r, int b_theta, int m, int64_t capacity) {
  Layout L{};
  L.d = d;
  L.pairs = d / 2;
  L.b_r = b_r;
  L.b_theta = b_theta;
  L.bw = b_r + b_theta;
  L.m = m;
  L.kc_bytes = L.pairs * L.bw / 8;
  L.sg_bytes = m / 8;
  L.pt = L.pairs / 4;
  L.kwt = words_for_bits(2 * L.pt * L.bw);
  L.sw = words_for_bits(2 * (m / 4));
  L.vwt = L.kwt;
  L.off_kc = 0;
  L.off_ks = L.off_kc + 128 * L.kwt;
  L.off_ksc = L.off_ks + 128 * L.sw;
  L.off_vc = L.off_ksc + 64;
  L.off_vsc = L.off_vc + 128 * L.vwt;
  L.tile_bytes = L.off_vsc + 32;
  L.block_bytes = kTilesPerBlock * L.tile_bytes;
  L.blocks_per_unit = (capacity + kTokensPerBlock - 1) / kTokensPerBlock;
  return L;
}


// ---- ragged batches: per-row lengths -------------------------------------
// When the rows of a batch hold different numbers of cold or hot tokens,
// the kernels read each row's counts from this table (in the workspace,
// written by one small launch whenever the counts change).
constexpr int kMaxRaggedRows = 128;

struct RowTable {
  int32_t n_cold[kMaxRaggedRows];         // cold tokens of row b (before an append / insert)
  int32_t n_hot[kMaxRaggedRows];          // valid hot tokens
  int32_t ring_pos[kMaxRaggedRows];       // next ring slot
  int32_t n_new[kMaxRaggedRows];          // tokens the current append / insert brings to row b
  int32_t cold_pre[kMaxRaggedRows + 1];   // (decode) cold blocks of the units of rows before b
  int32_t hot_pre[kMaxRaggedRows + 1];    // (decode) hot tiles of the units of rows before b
};

cudaError_t launch_rows_upload(RowTable* dst, const RowTable& src, cudaStream_t s);

// ---- attention-weighted promotion ---------------------------------------
// At most this many tokens per (row, kv head) are counted or promoted per
// decode step: with a threshold >= 1/8 no more can reach it, because a
// unit's cold masses sum to at most 1.
constexpr int kPromoMax = 8;

// Per-(row, kv head) state in the caller's promotion buffer (128 bytes).
struct PromoUnitState {
  int cnt_idx[kPromoMax];   // cold positions with a running count (ascending), -1 unused
  int cnt_val[kPromoMax];
  int n_cnt;
  int pend_idx[kPromoMax];  // promoted by the last decode, not yet in the ring (ascending)
  int n_pend;
  int ring_pos;             // next ring slot of this unit
  int pad[5];
};

// ---- encode -------------------------------------------------------------
// Encodes a sequence of E vectors per unit (unit = row * Hkv + kv head), K
// and V in one launch: the first nA come from ring slots (ring_start + e)
// mod W, the next nB from source tokens 0..nB-1 ([units, src_tokens, d]).
// Vector e is stored at cold index cold_start + e.
struct EncodeArgs {
  const __half* ring_k;     // [units, W, d] or null
  const __half* ring_v;
  int W;
  int ring_start;
  int nA;
  const __half* src_k;      // [units, src_tokens, d] or null
  const __half* src_v;
  int64_t src_tokens;
  int64_t nB;
  uint8_t* cold;
  int64_t cold_start;
  int units;
  Layout L;
  const double* signs;      // [d]
  const float* St;          // S transposed, [d, m]
  const float* Stl;         // S^T by lane: [d][32][ceil(m/32)], element (j, l, k) = S^T[j][l + 32 k]
  const double2* atab;      // angle tables (angle_table_host)
  int* status;
  double inv_sqrt_d;        // 1 / sqrt(d), correctly rounded on the host
  // Steady-state eviction (per-token path only): after reading ring slot
  // (ring_start + e) mod W, token e's CTA writes src_k/src_v token e into
  // that same slot, so the ring write needs no launch of its own.
  int write_new;
  // Eviction with promotion (per-token path; null otherwise): unit u
  // inserts its n_pend promoted tokens (promo_k/v) and then n_new new ones
  // (src) at its own ring position; insert e evicts ring slot (ring_pos +
  // e) mod W into cold position pend_idx[e] (e < n_pend) or cold_start +
  // e - n_pend, and takes that slot.
  const PromoUnitState* promo;
  const __half* promo_k;
  const __half* promo_v;
  int n_new;
  // Ragged batch (null otherwise): row b = unit / Hkv appends rows->n_new[b]
  // tokens at rows->n_cold[b] (ring_k null), or inserts them into its ring
  // (evicting max(0, n_hot + n_new - W) tokens, the ring's oldest first);
  // source tokens are [units, src_tokens = n_max, d].  groups_max: the most
  // 4-token groups of 16-token tiles any unit writes (warp path).
  const RowTable* rows;
  int Hkv;
  int n_max;
  int64_t groups_max;
};

// Global -> shared copy of `bytes` (a multiple of 16, both addresses 16-byte
// aligned) as asynchronous 16-byte copies spread over the block's threads:
// no thread waits for them here.  Before reading, every thread calls
// async_copy_wait() (its own copies) and the block meets at a barrier.
__device__ __forceinline__ void async_copy_g2s(void* dst, const void* src, int bytes) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  for (int i = (int)threadIdx.x * 16; i < bytes; i += (int)blockDim.x * 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d + i),
                 "l"(reinterpret_cast<const char*>(src) + i)
                 : "memory");
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

__device__ __forceinline__ void async_copy_wait() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// Appends of up to this many tokens per unit take the per-token (latency)
// encode path; longer ones the warp-per-vector (throughput) path.
constexpr int64_t kSmallEncodeTokens = 8;

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s);

// Copies new tokens i in [first, n) into ring slots (ring_pos + i) mod W
// (ragged: row b's tokens i in [max(0, n_new - W), n_new) at its own ring
// position, from [units, n, d]).
cudaError_t launch_ring_write(__half* ring_k, __half* ring_v, const __half* k_new,
                              const __half* v_new, int units, int W, int d, int n,
                              int first, int ring_pos, cudaStream_t s,
                              const RowTable* rows = nullptr, int Hkv = 1);

// ---- decode -------------------------------------------------------------
// Query transforms of one decode call (written by q-prep, per query head h):
//   qrot   [h][2][d]       q' * a1 as fp16 hi and lo parts (a1 a power of 2)
//   qk8    [h][2][d/16][32] int8 planes (hi, lo) of the projections of q'
//                          on the slot directions, in int8 B-fragment order
//   qs8    [h][2][m/32][32] int8 planes of q'' = S q', B-fragment order
//   qscale [h][4]          1/a1, alpha_k, alpha_s (the planes' value of one
//                          unit: x = alpha (256 hi + lo)), and the integer
//                          sum of q'' / alpha_s (int32 bits)
// Byte (plane, s, t, 4 hf + e) of qk8 is slot e of pair t * d/8 + 2 s + hf;
// of qs8 it is sign t * m/4 + 8 s + 4 hf + e.
struct QBufs {
  __half* qrot;
  int8_t* qk8;
  int8_t* qs8;
  float* qscale;
};

// Offsets of the query transforms in a scratch area (256-byte aligned).
struct QBufsLayout {
  size_t qrot, qk8, qs8, qscale, total;
};

inline QBufsLayout qbufs_layout(size_t heads, int d, int m) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  QBufsLayout l{};
  size_t off = 0;
  l.qrot = off;   off += up(heads * 2 * d * 2);
  l.qk8 = off;    off += up(heads * 2 * (d / 16) * 32);
  l.qs8 = off;    off += up(heads * 2 * (m / 32) * 32);
  l.qscale = off; off += up(heads * 4 * sizeof(float));
  l.total = off;
  return l;
}

inline QBufs qbufs_at(uint8_t* base, const QBufsLayout& l) {
  return QBufs{(__half*)(base + l.qrot), (int8_t*)(base + l.qk8), (int8_t*)(base + l.qs8),
               (float*)(base + l.qscale)};
}

struct QPrepArgs {
  const __half* q;          // [B*Hq, d]
  const double* signs;      // [d]
  const float* St;          // [d, m]
  QBufs out;
  int heads;                // B*Hq
  int d, m;
  int b_theta;              // slot directions: 2^(b_theta-1) (b_theta <= 3), else unused
};

cudaError_t launch_qprep(const QPrepArgs& a, cudaStream_t s);

// Work partition of one decode call.  The cold blocks of all units form one
// flattened list (unit-major); cold CTA c takes blocks [c*cold_bpc,
// (c+1)*cold_bpc) of it and writes one partial per unit it touches, into
// slot c - first_cta(unit).  Hot tiles are split the same way by hot CTAs,
// whose partials follow the cold slots.
constexpr int kSlotsCold = 96;     // partial slots per (row, kv head) for cold CTAs
constexpr int kSlotsHot = 32;      // ... and for hot CTAs

struct SplitPlan {
  int64_t cold_blocks;      // 64-token blocks holding valid cold tokens, per unit
  int cold_ctas;
  int64_t cold_bpc;         // blocks per cold CTA
  int hot_tiles;            // 64-token hot tiles per unit
  int hot_ctas;
  int hot_tpc;              // tiles per hot CTA
  int slots_cold;           // partial slots per unit reserved for cold CTAs
  int slots_hot;
};

// Cold split of a gated decode call, over the n_active units whose cold
// tier is read: blocks per CTA as in the host plan (at least enough that a
// unit spans at most kSlotsCold - 1 CTAs), for at most `ctas_max` CTAs (the
// launch's cold CTAs when every unit is read).
__host__ __device__ inline void gated_cold_split(int64_t n_active, int64_t nb, int ctas_max,
                                                 int64_t* bpc, int* ctas) {
  const int64_t total = n_active * nb;
  int64_t b = ctas_max > 0 ? (total + ctas_max - 1) / ctas_max : 1;
  const int64_t lo = nb > 1 ? (nb - 1 + kSlotsCold - 3) / (kSlotsCold - 2) : 1;
  if (b < lo) b = lo;
  *bpc = b;
  *ctas = (int)((total + b - 1) / b);
}

// Partial record per (unit, slot, head): {m (log2 units), l, o[d]}.
struct AttendArgs {
  const __half* q;          // [B*Hq, d]  (hot logits use q itself)
  const __half* qrot;       // query transforms (QBufs)
  const int8_t* qk8;
  const int8_t* qs8;
  const float* qscale;
  const __half* hot_k;      // [units, W, d]
  const __half* hot_v;
  const uint8_t* cold;
  float* part;              // [units, slots_cold + slots_hot, G, d + 2]
  int* status;
  Layout L;
  SplitPlan plan;
  int units, G, Hq, Hkv;
  int W, n_hot;
  int64_t n_cold;
  float log2e_sigma;        // log2(e) * softmax scale
  // Ragged batch (the attention kernel's RAGGED mode): per-row counts and
  // the units' block / tile prefix sums.
  const RowTable* rows;
  // When non-null (promotion enabled): every valid cold token's log2-domain
  // logit of every query head, [units][logit_capacity][G].
  float* logits;
  int64_t logit_capacity;
  // Limit of each bounded wait for a cold tile's bulk copy; 0 makes every
  // such wait give up at once (a forced timeout).  The copies already issued
  // are then drained under kDefaultWaitLimitNs before the CTA exits.
  unsigned long long wait_limit_ns;
  // gated calls only (null otherwise): the units whose cold tier is read,
  // in unit order, and their count (written by gate_kernel)
  const int* alist;         // [units + 1]
  const int* n_active;
};

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s);
int attend_ctas_per_sm(const Layout& L, int G);

struct CombineArgs {
  const float* part;
  const RowTable* rows;     // ragged batch, or null
  float* ml;                // null, or [B*Hq][2]: each head's final max (log2) and sum
  const int* status;        // device status word: NaN output while kStatusNoPartials is latched
  const double* signs;
  float* out;               // [B*Hq, d]
  SplitPlan plan;
  int units, G, Hkv, Hq, d, batch;
  // gated calls only (null otherwise)
  const int* head_skip;     // [B*Hq]  1: the head's cold partials are left out
  const int* unit_pos;      // [units] position in the active list, or -1
  const int* n_active;
};

// Threshold gate of the cold tier: per query head, the largest plain score
// q.k over the hot window; the head skips its cold tier when the window is
// non-empty and that score is at least `threshold`.  Block c of a unit
// writes its per-head maxima of rows [c * rows, (c + 1) * rows) to cmax;
// the last block to finish reduces them, takes the decisions and lists the
// units with at least one head that reads its cold tier.
constexpr int kGateRowsMin = 128;   // fewest hot rows a gate block takes (d = 128)

struct GateArgs {
  const __half* q;          // [B*Hq, d]
  const __half* hot_k;      // [units, W, d]
  int* head_skip;           // [B*Hq]
  float* cmax;              // [B*Hq, chunks]  per-block maxima
  int* unit_pos;            // [units]
  int* alist;               // [units + 1]
  int* n_active;
  unsigned* counter;        // 0 between calls
  int units, G, Hq, Hkv, W, n_hot, d;
  int dirty_lo, dirty_n;    // ring slots [lo, lo + n) mod W written by the last eviction
  float threshold;
};

cudaError_t launch_gate(const GateArgs& a, cudaStream_t s);

// ---- promotion kernels --------------------------------------------------
struct PromoArgs {
  const float* logits;      // [units][capacity][G] log2-domain logits of the last decode
  const float* ml;          // [B*Hq][2] each head's final max (log2) and sum
  PromoUnitState* state;    // [units]
  const uint8_t* cold;
  __half* promo_k;          // [units][kPromoMax][d] dequantized promoted tokens
  __half* promo_v;
  const double* signs;
  double inv_sqrt_d;
  Layout L;
  int units, G, Hq, Hkv;
  int64_t n_cold, capacity;
  float threshold;
  int sticky;
  int ring_full;            // promotions are kept only while the hot window is full
};

cudaError_t launch_promo_mass(const PromoArgs& a, cudaStream_t s);
cudaError_t launch_promo_dequant(const PromoArgs& a, cudaStream_t s);
cudaError_t launch_promo_ring(PromoUnitState* state, int units, int W, int n_new, int set_to,
                              cudaStream_t s);

// ---- Tensor Cache second tier -----------------------------------------
// Per unit a d x d float32 matrix A; per kv head lambda, eta; per query
// head sigmoid(g).  Evicted tokens e = 0 .. E-1 (oldest first: nA ring
// slots from ring_start, then the first nB new tokens) are written as
// A <- lambda^E A + eta sum_e lambda^(E-1-e) k_e v_e^T, which equals E
// sequential writes A <- lambda A + eta k_e v_e^T.
struct TcUpdateArgs {
  float* A;                 // [units, d, d]
  const float* lam;         // [Hkv]
  const float* eta;         // [Hkv]
  const __half* ring_k;     // [units, W, d]
  const __half* ring_v;
  const __half* src_k;      // [units, src_tokens, d]
  const __half* src_v;
  int units, Hkv, W, d;
  int nA, ring_start;
  int nB, src_tokens;
};

// out[h] += sigmoid(g_h) (q_h A_unit) for every query head h.
struct TcReadArgs {
  const float* A;           // [units, d, d]
  const float* sig;         // [Hq]  sigmoid(g)
  const __half* q;          // [B*Hq, d]
  float* out;               // [B*Hq, d]
  int units, G, Hq, d;
};

cudaError_t launch_tc_update(const TcUpdateArgs& a, cudaStream_t s);
cudaError_t launch_tc_read(const TcReadArgs& a, cudaStream_t s);

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

// ---- vector search ----------------------------------------------------
struct VecEncodeArgs {
  const float* x;           // [count, dim]
  int64_t start, count;
  int dim;
  Layout L;                 // d (padded), b_r, b_theta, m
  const double* signs;
  const float* St;          // [d, m]
  const double2* atab;      // angle tables (angle_table_host)
  double inv_sqrt_d;
  int* status;
  uint8_t* codes;           // [n/32][d/32][32][16 B]: 32-vector groups, 16-byte chunks
  uint8_t* signs_out;       // [n/32][2][32][16 B]
  uint16_t* s16_out;        // [n]
  uint16_t* rn16_out;       // [n]
};

struct VecQPrepArgs {
  const float* q;           // [nq, dim]
  int nq, dim, d, m;
  const double* signs;
  const float* St;
  int kq;                   // QJL k-steps of 16 (search_qjl_steps)
  int half_last;            // the last QJL k-step takes the high half of its word only
  __half* A;                // query tiles of 128 rows, UMMA core-matrix order
  float* qscale;            // [nq]
};

struct SearchArgs {
  const __half* A;
  const uint8_t* codes;
  const uint8_t* signs;
  const uint16_t* s16;
  const uint16_t* rn16;
  int64_t n;
  int nq, d, b_theta, nsplit;
  int kq, half_last;        // as in VecQPrepArgs
  float inv_levels;         // 1 / (2^b_r - 1)
  float qjl_const;          // sqrt(pi/2) / m
  float* part_s;            // [nq][nsplit][16]
  int* part_i;
  int* status;              // latched kStatusTimeout
  unsigned long long wait_limit_ns;
};

struct MergeArgs {
  const float* part_s;
  const int* part_i;
  const float* qscale;
  int nq, nsplit, k;
  float* scores;            // [nq, k]
  int* idx;
};

cudaError_t launch_vec_encode(const VecEncodeArgs& a, cudaStream_t s);
cudaError_t launch_vec_qprep(const VecQPrepArgs& a, cudaStream_t s);
cudaError_t launch_search(const SearchArgs& a, cudaStream_t s);
cudaError_t launch_topk_merge(const MergeArgs& a, cudaStream_t s);

}  // namespace tq
