// C-ABI entry points of the compressed KV-cache library: argument checks,
// buffer layout, the seeded method randomness (rotation signs D, QJL matrix
// S) and the launch sequence of each call.  See include/tq.h for the
// contract of every function.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- seeded generator (SplitMix64 finalizer over a Weyl sequence) --------
// Steele, Lea & Flood, "Fast splittable pseudorandom number generators"
// (OOPSLA 2014): mix64 is the SplitMix64 output function.
uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t rand64(uint64_t seed, uint64_t stream, uint64_t i) {
  const uint64_t base = mix64(seed + stream);
  return mix64(base + (i + 1) * 0x9E3779B97F4A7C15ull);
}

void gen_signs(uint64_t seed, int d, double* out) {
  for (int i = 0; i < d; ++i) out[i] = (rand64(seed, 0, (uint64_t)i) >> 63) ? -1.0 : 1.0;
}

void gen_qjl(uint64_t seed, int m, int d, float* out) {
  const double two_pi = 2.0 * M_PI;
  const double scale = 1.0 / 9007199254740992.0;  // 2^-53
  const uint64_t total = (uint64_t)m * (uint64_t)d;
  for (uint64_t k = 0; k < total; ++k) {
    const uint64_t a = rand64(seed, 1, 2 * k);
    const uint64_t b = rand64(seed, 1, 2 * k + 1);
    const double u1 = (double)((a >> 11) + 1) * scale;
    const double u2 = (double)(b >> 11) * scale;
    const double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
    out[k] = (float)z;
  }
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

}  // namespace

struct WsLayout {
  size_t status, signs, Stl, St, atab, q, part, gate, gate_max, rows, total;
  QBufsLayout ql;               // query transforms, at offset q
};

static WsLayout ws_layout(const tq_config& c) {
  WsLayout w{};
  const size_t heads = (size_t)c.batch * c.num_q_heads;
  const size_t units = (size_t)c.batch * c.num_kv_heads;
  const size_t G = (size_t)(c.num_q_heads / c.num_kv_heads);
  size_t off = 0;
  w.status = off; off += kAlign;
  w.signs = off;  off += round_up(sizeof(double) * c.head_dim, kAlign);
  w.Stl = off;    off += round_up(sizeof(float) * c.head_dim * 32 * ((c.qjl_bits + 31) / 32), kAlign);
  w.St = off;     off += round_up(sizeof(float) * c.head_dim * c.qjl_bits, kAlign);
  w.atab = off;   off += round_up(sizeof(double) * 2 * kAngleTableEntries, kAlign);
  w.ql = qbufs_layout(heads, c.head_dim, c.qjl_bits);
  w.q = off;      off += w.ql.total;
  w.part = off;   off += round_up(sizeof(float) * units * (kSlotsCold + kSlotsHot) * G * (c.head_dim + 2), kAlign);
  // gated decode: head_skip [heads], unit_pos [units], alist [units + 1], n_active, then the
  // gate blocks' maxima [heads, ceil(W / kGateRowsMin)]
  const size_t gate_chunks = (c.hot_window + kGateRowsMin - 1) / kGateRowsMin;
  w.gate = off;   off += round_up(sizeof(int) * (heads + 2 * units + 2), kAlign);
  w.gate_max = off; off += round_up(sizeof(float) * heads * std::max<size_t>(gate_chunks, 1), kAlign);
  w.rows = off;   off += round_up(sizeof(RowTable), kAlign);   // per-row counts of a ragged batch
  w.total = off;
  return w;
}

static tq_status check_config(const tq_config* c) {
  if (!c) return TQ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->num_q_heads < 1 || c->num_kv_heads < 1 || c->hot_window < 1 ||
      c->cold_capacity < 0 || c->b_r < 1 || c->b_theta < 1 || c->qjl_bits < 8 ||
      c->head_dim < 2 || (c->qjl_bits % 8) != 0 || !is_pow2(c->head_dim))
    return TQ_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads != 0) return TQ_ERR_INVALID_ARG;
  if (c->b_r + c->b_theta > 8) return TQ_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return TQ_ERR_UNSUPPORTED;
  if (c->qjl_bits != 64 && c->qjl_bits != 128) return TQ_ERR_UNSUPPORTED;
  if (c->num_q_heads / c->num_kv_heads > 8) return TQ_ERR_UNSUPPORTED;
  return TQ_OK;
}

}  // namespace tq

using namespace tq;

struct tq_cache {
  tq_config cfg;
  Layout L;
  WsLayout W;
  uint8_t* hot;
  uint8_t* cold;
  uint8_t* ws;
  int64_t n_cold;
  int32_t n_hot;
  int32_t ring_pos;
  int32_t dirty_lo, dirty_n;   // ring slots the last tq_evict_window wrote
  float* tc;                   // Tensor Cache tier: A [units, d, d], or null
  float* tc_lam;               // [Hkv]
  float* tc_eta;               // [Hkv]
  float* tc_sig;               // [Hq] sigmoid(g)
  int num_sms;
  int ctas_per_sm;
  int device;
  cudaEvent_t ev_start;
  cudaEvent_t ev_stop;
  unsigned long long wait_limit_ns;   // attention kernel's bounded waits (tq_set_wait_limit)
  // per batch row: cold tokens, valid hot tokens, next ring slot.  While
  // they are equal across rows (`ragged` false) the scalars above hold them
  // and the uniform paths run; otherwise the kernels read a RowTable.
  std::vector<int64_t> row_cold;
  std::vector<int32_t> row_hot, row_pos;
  bool ragged;
  // attention-weighted promotion (tq_promotion_enable), or null
  uint8_t* promo;
  float promo_threshold;
  int promo_sticky;
  __half* hot_k() const { return (__half*)hot; }
  __half* hot_v() const {
    return (__half*)(hot + (size_t)cfg.batch * cfg.num_kv_heads * cfg.hot_window * cfg.head_dim * 2);
  }
  int* status() const { return (int*)(ws + W.status); }
  double* signs() const { return (double*)(ws + W.signs); }
  float* Stl() const { return (float*)(ws + W.Stl); }
  double2* atab() const { return (double2*)(ws + W.atab); }
  float* St() const { return (float*)(ws + W.St); }
};

// Promotion buffer: per-unit state | logits [units][capacity][G] fp32 |
// per-head (max, sum) | dequantized promoted tokens [units][8][2][d] fp16.
struct PromoLayout {
  size_t state, logits, ml, staging, total;
};

static PromoLayout promo_layout(const tq_config& c) {
  const size_t units = (size_t)c.batch * c.num_kv_heads;
  const size_t G = (size_t)(c.num_q_heads / c.num_kv_heads);
  PromoLayout p{};
  size_t off = 0;
  p.state = off;   off += round_up(sizeof(PromoUnitState) * units, kAlign);
  p.logits = off;  off += round_up(sizeof(float) * units * (size_t)c.cold_capacity * G, kAlign);
  p.ml = off;      off += round_up(sizeof(float) * 2 * (size_t)c.batch * c.num_q_heads, kAlign);
  p.staging = off; off += round_up(2 * units * kPromoMax * 2 * (size_t)c.head_dim, kAlign);
  p.total = off;
  return p;
}

static PromoArgs promo_args(const tq_cache* c) {
  const tq_config& cf = c->cfg;
  const PromoLayout pl = promo_layout(cf);
  const size_t units = (size_t)cf.batch * cf.num_kv_heads;
  PromoArgs a{};
  a.logits = (const float*)(c->promo + pl.logits);
  a.ml = (const float*)(c->promo + pl.ml);
  a.state = (PromoUnitState*)(c->promo + pl.state);
  a.cold = c->cold;
  a.promo_k = (__half*)(c->promo + pl.staging);
  a.promo_v = a.promo_k + units * kPromoMax * cf.head_dim;
  a.signs = c->signs();
  a.inv_sqrt_d = 1.0 / std::sqrt((double)cf.head_dim);
  a.L = c->L;
  a.units = (int)units;
  a.G = cf.num_q_heads / cf.num_kv_heads;
  a.Hq = cf.num_q_heads;
  a.Hkv = cf.num_kv_heads;
  a.n_cold = c->n_cold;
  a.capacity = cf.cold_capacity;
  a.threshold = c->promo_threshold;
  a.sticky = c->promo_sticky;
  a.ring_full = c->n_hot == cf.hot_window;
  return a;
}

// ---- per-row state -----------------------------------------------------
// After a uniform operation every row takes the scalars' values; after a
// ragged one the scalars are set from the rows when those agree again.
static void rows_from_scalars(tq_cache* c) {
  std::fill(c->row_cold.begin(), c->row_cold.end(), c->n_cold);
  std::fill(c->row_hot.begin(), c->row_hot.end(), c->n_hot);
  std::fill(c->row_pos.begin(), c->row_pos.end(), c->ring_pos);
}

static void scalars_from_rows(tq_cache* c) {
  const int B = c->cfg.batch;
  bool same = true;
  for (int b = 1; b < B; ++b)
    same &= c->row_cold[b] == c->row_cold[0] && c->row_hot[b] == c->row_hot[0] &&
            c->row_pos[b] == c->row_pos[0];
  c->ragged = !same;
  c->n_cold = *std::max_element(c->row_cold.begin(), c->row_cold.end());
  c->n_hot = *std::max_element(c->row_hot.begin(), c->row_hot.end());
  c->ring_pos = c->row_pos[0];
  c->dirty_lo = 0;
  c->dirty_n = c->cfg.hot_window;      // the gate reads the whole window after a ragged step
}

// The row table of the current counts (n_new per row, and the decode's
// prefix sums of blocks / tiles), written into the workspace.
static RowTable build_rows(const tq_cache* c, const int32_t* n_new) {
  const int B = c->cfg.batch, H = c->cfg.num_kv_heads;
  RowTable t{};
  t.cold_pre[0] = t.hot_pre[0] = 0;
  for (int b = 0; b < B; ++b) {
    t.n_cold[b] = (int32_t)c->row_cold[b];
    t.n_hot[b] = c->row_hot[b];
    t.ring_pos[b] = c->row_pos[b];
    t.n_new[b] = n_new ? n_new[b] : 0;
    t.cold_pre[b + 1] = t.cold_pre[b] + H * (int32_t)((c->row_cold[b] + kTokensPerBlock - 1) / kTokensPerBlock);
    t.hot_pre[b + 1] = t.hot_pre[b] + H * ((c->row_hot[b] + kTokensPerBlock - 1) / kTokensPerBlock);
  }
  return t;
}

static tq_status upload_rows(tq_cache* c, const int32_t* n_new, cudaStream_t stream, RowTable* out = nullptr) {
  const RowTable t = build_rows(c, n_new);
  if (out) *out = t;
  if (launch_rows_upload((RowTable*)(c->ws + c->W.rows), t, stream) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

extern "C" {

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CAPACITY: return "TQ_ERR_CAPACITY";
    case TQ_ERR_RANGE: return "TQ_ERR_RANGE";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
  }
  return "TQ_UNKNOWN";
}

int32_t tq_abi_version(void) { return TQ_ABI_VERSION; }

tq_status tq_cache_bytes(const tq_config* cfg, size_t* hot_bytes, size_t* cold_bytes,
                         size_t* workspace_bytes) {
  tq_status st = check_config(cfg);
  if (st != TQ_OK) return st;
  const Layout L = layout_of(cfg->head_dim, cfg->b_r, cfg->b_theta, cfg->qjl_bits,
                               cfg->cold_capacity);
  const size_t units = (size_t)cfg->batch * cfg->num_kv_heads;
  if (hot_bytes) *hot_bytes = 2 * units * cfg->hot_window * cfg->head_dim * 2;
  if (cold_bytes) *cold_bytes = units * (size_t)L.blocks_per_unit * L.block_bytes;
  if (workspace_bytes) *workspace_bytes = ws_layout(*cfg).total;
  return TQ_OK;
}

tq_status tq_cache_create(const tq_config* cfg, void* hot_mem, void* cold_mem,
                          void* workspace_mem, cudaStream_t stream, tq_cache** out) {
  tq_status st = check_config(cfg);
  if (st != TQ_OK) return st;
  if (!out || !hot_mem || !workspace_mem || (!cold_mem && cfg->cold_capacity > 0))
    return TQ_ERR_INVALID_ARG;
  if (((uintptr_t)hot_mem | (uintptr_t)cold_mem | (uintptr_t)workspace_mem) % kAlign)
    return TQ_ERR_INVALID_ARG;
  tq_cache* c = new (std::nothrow) tq_cache();
  if (!c) return TQ_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->L = layout_of(cfg->head_dim, cfg->b_r, cfg->b_theta, cfg->qjl_bits, cfg->cold_capacity);
  c->W = ws_layout(*cfg);
  c->hot = (uint8_t*)hot_mem;
  c->cold = (uint8_t*)cold_mem;
  c->ws = (uint8_t*)workspace_mem;
  c->n_cold = 0;
  c->n_hot = 0;
  c->ring_pos = 0;
  c->dirty_lo = 0;
  c->dirty_n = 0;
  c->tc = c->tc_lam = c->tc_eta = c->tc_sig = nullptr;
  c->wait_limit_ns = kDefaultWaitLimitNs;
  c->promo = nullptr;
  c->row_cold.assign(cfg->batch, 0);
  c->row_hot.assign(cfg->batch, 0);
  c->row_pos.assign(cfg->batch, 0);
  c->ragged = false;
  if (cudaGetDevice(&c->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
    delete c;
    return TQ_ERR_CUDA;
  }
  c->ctas_per_sm = attend_ctas_per_sm(c->L, cfg->num_q_heads / cfg->num_kv_heads);
  if (c->ctas_per_sm <= 0) {
    delete c;
    return TQ_ERR_CUDA;
  }
  const int d = cfg->head_dim, m = cfg->qjl_bits;
  std::vector<double> signs(d);
  const int nk = (m + 31) / 32;
  std::vector<float> S((size_t)m * d), St((size_t)m * d), Stl((size_t)d * 32 * nk, 0.f);
  gen_signs(cfg->seed, d, signs.data());
  gen_qjl(cfg->seed, m, d, S.data());
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      St[(size_t)j * m + i] = S[(size_t)i * d + j];
      Stl[((size_t)j * 32 + i % 32) * nk + i / 32] = S[(size_t)i * d + j];
    }
  // Pageable sources: cudaMemcpyAsync returns once the data is staged, so
  // the vectors may be released when the calls return.
  cudaError_t e = cudaMemsetAsync(c->status(), 0, kAlign, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->signs(), signs.data(), sizeof(double) * d, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->Stl(), Stl.data(), sizeof(float) * Stl.size(), cudaMemcpyHostToDevice, stream);
  std::vector<double> atab(2 * kAngleTableEntries, 0.0);
  angle_table_host(1 << cfg->b_theta, atab.data());
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->atab(), atab.data(), sizeof(double) * atab.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->St(), St.data(), sizeof(float) * St.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    delete c;
    return TQ_ERR_CUDA;
  }
  *out = c;
  return TQ_OK;
}

tq_status tq_cache_destroy(tq_cache* cache) {
  delete cache;
  return TQ_OK;
}

tq_status tq_cache_counts(const tq_cache* c, int64_t* n_cold, int32_t* n_hot, int32_t* ring_pos) {
  if (!c) return TQ_ERR_INVALID_ARG;
  if (n_cold) *n_cold = c->n_cold;
  if (n_hot) *n_hot = c->n_hot;
  if (ring_pos) *ring_pos = c->ring_pos;
  return TQ_OK;
}

static EncodeArgs base_encode_args(tq_cache* c) {
  EncodeArgs a{};
  a.W = c->cfg.hot_window;
  a.cold = c->cold;
  a.cold_start = c->n_cold;
  a.units = c->cfg.batch * c->cfg.num_kv_heads;
  a.L = c->L;
  a.signs = c->signs();
  a.St = c->St();
  a.Stl = c->Stl();
  a.atab = c->atab();
  a.status = c->status();
  a.inv_sqrt_d = 1.0 / std::sqrt((double)c->cfg.head_dim);
  return a;
}

// Append n tokens to every row (rows share their counts); source tokens
// are [units, src_tokens, d].
static tq_status encode_append_uniform(tq_cache* c, const void* k, const void* v, int64_t n,
                                       int64_t src_tokens, cudaStream_t stream) {
  if (n == 0) return TQ_OK;
  if (!k || !v) return TQ_ERR_INVALID_ARG;
  if (c->n_cold + n > c->cfg.cold_capacity) return TQ_ERR_CAPACITY;
  EncodeArgs a = base_encode_args(c);
  a.src_k = (const __half*)k;
  a.src_v = (const __half*)v;
  a.src_tokens = src_tokens;
  a.nB = n;
  a.nA = 0;
  if (launch_encode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  c->n_cold += n;
  return TQ_OK;
}

// Insert n tokens into every row's ring (rows share their counts).
static tq_status evict_window_uniform(tq_cache* c, const void* k_new, const void* v_new, int32_t n,
                                      cudaStream_t stream) {
  const int W = c->cfg.hot_window;
  const int64_t E = std::max<int64_t>(0, (int64_t)c->n_hot + n - W);
  if (c->tc) {
    // Tensor Cache tier: the displaced tokens are written into A (before
    // the ring write overwrites their slots); the cold store is untouched
    if (E > 0) {
      TcUpdateArgs t{};
      t.A = c->tc;
      t.lam = c->tc_lam;
      t.eta = c->tc_eta;
      t.ring_k = c->hot_k();
      t.ring_v = c->hot_v();
      t.src_k = (const __half*)k_new;
      t.src_v = (const __half*)v_new;
      t.units = c->cfg.batch * c->cfg.num_kv_heads;
      t.Hkv = c->cfg.num_kv_heads;
      t.W = W;
      t.d = c->cfg.head_dim;
      t.nA = (int)std::min<int64_t>(E, c->n_hot);
      t.ring_start = ((c->ring_pos - c->n_hot) % W + W) % W;
      t.nB = (int)(E - t.nA);
      t.src_tokens = n;
      if (launch_tc_update(t, stream) != cudaSuccess) return TQ_ERR_CUDA;
    }
    const int first = std::max(0, n - W);
    if (launch_ring_write(c->hot_k(), c->hot_v(), (const __half*)k_new, (const __half*)v_new,
                          c->cfg.batch * c->cfg.num_kv_heads, W, c->cfg.head_dim, n, first,
                          c->ring_pos, stream) != cudaSuccess)
      return TQ_ERR_CUDA;
    c->n_hot = (int32_t)std::min<int64_t>(W, (int64_t)c->n_hot + n);
    c->dirty_lo = (int32_t)(((int64_t)c->ring_pos + first) % W);
    c->dirty_n = std::min(n, W);
    c->ring_pos = (int32_t)(((int64_t)c->ring_pos + n) % W);
    return TQ_OK;
  }
  if (c->n_cold + E > c->cfg.cold_capacity) return TQ_ERR_CAPACITY;
  if (c->promo && c->n_hot == W) {
    // Promotion enabled and the window full: unit u inserts its pending
    // promoted tokens, then the n new ones, at its own ring position; the
    // first evictions take the promoted tokens' cold positions, the last n
    // are appended (so every unit's cold count grows by n).
    if (n > W - kPromoMax) return TQ_ERR_INVALID_ARG;
    PromoArgs pa = promo_args(c);
    if (launch_promo_dequant(pa, stream) != cudaSuccess) return TQ_ERR_CUDA;
    EncodeArgs a = base_encode_args(c);
    a.ring_k = c->hot_k();
    a.ring_v = c->hot_v();
    a.src_k = (const __half*)k_new;
    a.src_v = (const __half*)v_new;
    a.src_tokens = n;
    a.promo = pa.state;
    a.promo_k = pa.promo_k;
    a.promo_v = pa.promo_v;
    a.n_new = n;
    if (launch_encode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
    if (launch_promo_ring(pa.state, pa.units, W, n, -1, stream) != cudaSuccess) return TQ_ERR_CUDA;
    c->n_cold += n;
    c->dirty_lo = 0;
    c->dirty_n = W;
    c->ring_pos = (int32_t)(((int64_t)c->ring_pos + n) % W);
    return TQ_OK;
  }
  // Steady state (a full window, a few new tokens): each new token evicts
  // the token in the slot it takes, and one launch does both.
  const bool fused = E == n && c->n_hot == W && n <= W && n <= kSmallEncodeTokens;
  if (E > 0) {
    EncodeArgs a = base_encode_args(c);
    a.nA = (int)std::min<int64_t>(E, c->n_hot);
    a.nB = E - a.nA;
    a.ring_k = c->hot_k();
    a.ring_v = c->hot_v();
    a.ring_start = ((c->ring_pos - c->n_hot) % W + W) % W;
    a.src_k = (const __half*)k_new;
    a.src_v = (const __half*)v_new;
    a.src_tokens = n;
    a.write_new = fused ? 1 : 0;
    if (launch_encode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  }
  if (!fused) {
    const int first = std::max(0, n - W);
    if (launch_ring_write(c->hot_k(), c->hot_v(), (const __half*)k_new, (const __half*)v_new,
                          c->cfg.batch * c->cfg.num_kv_heads, W, c->cfg.head_dim, n, first,
                          c->ring_pos, stream) != cudaSuccess)
      return TQ_ERR_CUDA;
  }
  c->n_cold += E;
  c->n_hot = (int32_t)std::min<int64_t>(W, (int64_t)c->n_hot + n);
  c->dirty_lo = (int32_t)(((int64_t)c->ring_pos + std::max(0, n - W)) % W);
  c->dirty_n = std::min(n, W);
  c->ring_pos = (int32_t)(((int64_t)c->ring_pos + n) % W);
  if (c->promo &&   // until the window is full every unit shares the host's ring position
      launch_promo_ring((PromoUnitState*)(c->promo + promo_layout(c->cfg).state),
                        c->cfg.batch * c->cfg.num_kv_heads, W, 0, c->ring_pos, stream) != cudaSuccess)
    return TQ_ERR_CUDA;
  return TQ_OK;
}

tq_status tq_encode_append(tq_cache* c, const void* k, const void* v, int64_t n, cudaStream_t stream) {
  if (!c || n < 0) return TQ_ERR_INVALID_ARG;
  if (c->ragged) {
    if (n > INT32_MAX) return TQ_ERR_INVALID_ARG;
    std::vector<int32_t> rows(c->cfg.batch, (int32_t)n);
    return tq_encode_append_rows(c, k, v, n, rows.data(), stream);
  }
  const tq_status st = encode_append_uniform(c, k, v, n, n, stream);
  if (st == TQ_OK) rows_from_scalars(c);
  return st;
}

tq_status tq_evict_window(tq_cache* c, const void* k_new, const void* v_new, int32_t n,
                          cudaStream_t stream) {
  if (!c || !k_new || !v_new || n < 1) return TQ_ERR_INVALID_ARG;
  if (c->ragged) {
    std::vector<int32_t> rows(c->cfg.batch, n);
    return tq_evict_window_rows(c, k_new, v_new, n, rows.data(), stream);
  }
  const tq_status st = evict_window_uniform(c, k_new, v_new, n, stream);
  if (st == TQ_OK) rows_from_scalars(c);
  return st;
}

// Most 4-token groups of 16-token tiles any row's units write when row b
// writes cold positions [n_cold_b, n_cold_b + cnt[b]).
static int64_t max_groups(const tq_cache* c, const std::vector<int64_t>& cnt) {
  int64_t g = 0;
  for (int b = 0; b < c->cfg.batch; ++b)
    if (cnt[b] > 0) {
      const int64_t s = c->row_cold[b], e = s + cnt[b] - 1;
      g = std::max<int64_t>(g, (e / kTokensPerTile - s / kTokensPerTile + 1) * 4);
    }
  return g;
}

tq_status tq_encode_append_rows(tq_cache* c, const void* k, const void* v, int64_t n_max,
                                const int32_t* n_rows, cudaStream_t stream) {
  if (!c || !n_rows || n_max < 0) return TQ_ERR_INVALID_ARG;
  const int B = c->cfg.batch;
  bool any = false, same = true;
  int64_t mx = 0;
  for (int b = 0; b < B; ++b) {
    if (n_rows[b] < 0 || n_rows[b] > n_max) return TQ_ERR_INVALID_ARG;
    any |= n_rows[b] > 0;
    same &= n_rows[b] == n_rows[0];
    mx = std::max<int64_t>(mx, n_rows[b]);
  }
  if (!any) return TQ_OK;
  if (!k || !v) return TQ_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (c->row_cold[b] + n_rows[b] > c->cfg.cold_capacity) return TQ_ERR_CAPACITY;
  if (same && !c->ragged) {
    const tq_status st = encode_append_uniform(c, k, v, n_rows[0], n_max, stream);
    if (st == TQ_OK) rows_from_scalars(c);
    return st;
  }
  if (B > kMaxRaggedRows || c->tc || c->promo) return TQ_ERR_UNSUPPORTED;
  if (upload_rows(c, n_rows, stream) != TQ_OK) return TQ_ERR_CUDA;
  EncodeArgs a = base_encode_args(c);
  a.src_k = (const __half*)k;
  a.src_v = (const __half*)v;
  a.src_tokens = n_max;
  a.rows = (const RowTable*)(c->ws + c->W.rows);
  a.Hkv = c->cfg.num_kv_heads;
  a.n_max = (int)mx;
  a.groups_max = max_groups(c, std::vector<int64_t>(n_rows, n_rows + B));
  if (launch_encode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  for (int b = 0; b < B; ++b) c->row_cold[b] += n_rows[b];
  scalars_from_rows(c);
  return TQ_OK;
}

tq_status tq_evict_window_rows(tq_cache* c, const void* k_new, const void* v_new, int32_t n_max,
                               const int32_t* n_rows, cudaStream_t stream) {
  if (!c || !n_rows || !k_new || !v_new || n_max < 1) return TQ_ERR_INVALID_ARG;
  const int B = c->cfg.batch, W = c->cfg.hot_window;
  bool any = false, same = true;
  std::vector<int64_t> ev(B);
  int64_t emax = 0;
  for (int b = 0; b < B; ++b) {
    if (n_rows[b] < 0 || n_rows[b] > n_max) return TQ_ERR_INVALID_ARG;
    any |= n_rows[b] > 0;
    same &= n_rows[b] == n_rows[0];
    ev[b] = std::max<int64_t>(0, (int64_t)c->row_hot[b] + n_rows[b] - W);
    emax = std::max(emax, ev[b]);
    if (c->row_cold[b] + ev[b] > c->cfg.cold_capacity) return TQ_ERR_CAPACITY;
  }
  if (!any) return TQ_OK;
  if (same && !c->ragged && n_rows[0] == n_max) {
    const tq_status st = evict_window_uniform(c, k_new, v_new, n_max, stream);
    if (st == TQ_OK) rows_from_scalars(c);
    return st;
  }
  if (B > kMaxRaggedRows || c->tc || c->promo) return TQ_ERR_UNSUPPORTED;
  if (upload_rows(c, n_rows, stream) != TQ_OK) return TQ_ERR_CUDA;
  const RowTable* rows = (const RowTable*)(c->ws + c->W.rows);
  if (emax > 0) {
    EncodeArgs a = base_encode_args(c);
    a.ring_k = c->hot_k();
    a.ring_v = c->hot_v();
    a.src_k = (const __half*)k_new;
    a.src_v = (const __half*)v_new;
    a.src_tokens = n_max;
    a.rows = rows;
    a.Hkv = c->cfg.num_kv_heads;
    a.n_max = (int)emax;
    a.groups_max = max_groups(c, ev);
    if (launch_encode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  }
  if (launch_ring_write(c->hot_k(), c->hot_v(), (const __half*)k_new, (const __half*)v_new,
                        B * c->cfg.num_kv_heads, W, c->cfg.head_dim, n_max, 0, 0, stream, rows,
                        c->cfg.num_kv_heads) != cudaSuccess)
    return TQ_ERR_CUDA;
  for (int b = 0; b < B; ++b) {
    c->row_cold[b] += ev[b];
    c->row_hot[b] = std::min(W, c->row_hot[b] + n_rows[b]);
    c->row_pos[b] = (int32_t)(((int64_t)c->row_pos[b] + n_rows[b]) % W);
  }
  scalars_from_rows(c);
  return TQ_OK;
}

tq_status tq_cache_row_counts(const tq_cache* c, int32_t row, int64_t* n_cold, int32_t* n_hot,
                              int32_t* ring_pos) {
  if (!c || row < 0 || row >= c->cfg.batch) return TQ_ERR_INVALID_ARG;
  if (n_cold) *n_cold = c->row_cold[row];
  if (n_hot) *n_hot = c->row_hot[row];
  if (ring_pos) *ring_pos = c->row_pos[row];
  return TQ_OK;
}

// Split plan: one wave of `ctas` CTAs.  Every CTA streams an equal run of
// the flattened (unit, cold block) list; CTAs [0, hot_ctas) then also take
// hot_tpc hot tiles each (one for the usual window sizes), so the latency
// of the fp16 hot tiles is paid once per CTA at the end of its cold run
// rather than by a few CTAs in turn.  `tight` sizes the partial slots per
// unit to the most any unit can receive under the plan (the static-scratch
// entry point); otherwise they are the workspace's fixed kSlotsCold /
// kSlotsHot.
static SplitPlan make_plan(int64_t n_cold, int n_hot, int units, int ctas, bool tight) {
  const int TB = kTokensPerBlock;
  const int64_t cold_blocks = (n_cold + TB - 1) / TB;
  const int hot_tiles = (n_hot + TB - 1) / TB;
  const int64_t N = (int64_t)units * cold_blocks;
  const int64_t Nh = (int64_t)units * hot_tiles;
  SplitPlan pl{};
  pl.cold_blocks = cold_blocks;
  pl.hot_tiles = hot_tiles;
  // tight: a side with no work reserves no slots (the kernels only use
  // slots below the counts they compute from the same plan)
  pl.slots_cold = tight ? 0 : kSlotsCold;
  pl.slots_hot = tight ? 0 : kSlotsHot;
  if (Nh > 0) {
    int64_t tpc = (Nh + ctas - 1) / ctas;
    // a unit's tiles may span at most kSlotsHot - 2 CTAs
    tpc = std::max<int64_t>(tpc, hot_tiles > 1 ? (hot_tiles - 1 + kSlotsHot - 3) / (kSlotsHot - 2) : 1);
    pl.hot_tpc = (int)tpc;
    pl.hot_ctas = (int)((Nh + tpc - 1) / tpc);
    if (tight) pl.slots_hot = (int)((hot_tiles - 1) / tpc + 2);
  }
  if (N > 0) {
    int64_t bpc = (N + ctas - 1) / ctas;
    bpc = std::max<int64_t>(bpc, cold_blocks > 1 ? (cold_blocks - 1 + kSlotsCold - 3) / (kSlotsCold - 2) : 1);
    pl.cold_bpc = bpc;
    pl.cold_ctas = (int)((N + bpc - 1) / bpc);
    if (tight) pl.slots_cold = (int)((cold_blocks - 1) / bpc + 2);
  }
  return pl;
}

// The split of a ragged batch: the units' blocks (tiles) are flattened by
// the table's prefix sums; blocks per CTA follow the uniform rule with the
// longest row's block count; `tight` sizes the slots to the most CTAs any
// unit spans.
static SplitPlan make_plan_ragged(const RowTable& t, int B, int H, int ctas, bool tight) {
  const int TB = kTokensPerBlock;
  int64_t maxnb = 0, maxht = 0;
  for (int b = 0; b < B; ++b) {
    maxnb = std::max<int64_t>(maxnb, (t.n_cold[b] + TB - 1) / TB);
    maxht = std::max<int64_t>(maxht, (t.n_hot[b] + TB - 1) / TB);
  }
  const int64_t N = t.cold_pre[B], Nh = t.hot_pre[B];
  SplitPlan pl{};
  pl.cold_blocks = maxnb;
  pl.hot_tiles = (int)maxht;
  pl.slots_cold = tight ? 0 : kSlotsCold;
  pl.slots_hot = tight ? 0 : kSlotsHot;
  auto span = [](int64_t off, int64_t n, int64_t per) { return n > 0 ? (int)((off + n - 1) / per - off / per + 1) : 0; };
  if (Nh > 0) {
    int64_t tpc = (Nh + ctas - 1) / ctas;
    tpc = std::max<int64_t>(tpc, maxht > 1 ? (maxht - 1 + kSlotsHot - 3) / (kSlotsHot - 2) : 1);
    pl.hot_tpc = (int)tpc;
    pl.hot_ctas = (int)((Nh + tpc - 1) / tpc);
    if (tight) {
      int mx = 0;
      for (int b = 0; b < B; ++b) {
        const int64_t ht = (t.n_hot[b] + TB - 1) / TB;
        for (int h = 0; h < H; ++h) mx = std::max(mx, span(t.hot_pre[b] + h * ht, ht, tpc));
      }
      pl.slots_hot = mx;
    }
  }
  if (N > 0) {
    int64_t bpc = (N + ctas - 1) / ctas;
    bpc = std::max<int64_t>(bpc, maxnb > 1 ? (maxnb - 1 + kSlotsCold - 3) / (kSlotsCold - 2) : 1);
    pl.cold_bpc = bpc;
    pl.cold_ctas = (int)((N + bpc - 1) / bpc);
    if (tight) {
      int mx = 0;
      for (int b = 0; b < B; ++b) {
        const int64_t nb = (t.n_cold[b] + TB - 1) / TB;
        for (int h = 0; h < H; ++h) mx = std::max(mx, span(t.cold_pre[b] + h * nb, nb, bpc));
      }
      pl.slots_cold = mx;
    }
  }
  return pl;
}

// Gated decode: the workspace's gate area and the caller's threshold.
struct GateBuffers {
  int* head_skip;
  float* cmax;
  int* unit_pos;
  int* alist;
  int* n_active;
  unsigned* counter;
  float threshold;
};

// The launches of one decode call: q-prep, the gate of the cold tier (gated
// calls only), the attention kernel (split partials), and the merge of the
// partials into the output rows.  Scratch buffers are the caller's
// (workspace or static scratch).
static tq_status launch_decode(tq_cache* c, const void* q, float* out, float softmax_scale,
                               const SplitPlan& pl, const QBufs& qb, float* part, cudaStream_t stream,
                               const GateBuffers* gate = nullptr, const RowTable* rows = nullptr) {
  const tq_config& cf = c->cfg;
  const int d = cf.head_dim;
  const int units = cf.batch * cf.num_kv_heads;
  const float sigma = softmax_scale == 0.0f ? (float)(1.0 / std::sqrt((double)d)) : softmax_scale;
  if (pl.cold_ctas == 0 && pl.hot_ctas == 0) {    // nothing cached: the output is zero
    if (cudaMemsetAsync(out, 0, sizeof(float) * cf.batch * cf.num_q_heads * d, stream) != cudaSuccess)
      return TQ_ERR_CUDA;
    return TQ_OK;
  }
  QPrepArgs qa{};
  qa.q = (const __half*)q;
  qa.signs = c->signs();
  qa.St = c->St();
  qa.out = qb;
  qa.heads = cf.batch * cf.num_q_heads;
  qa.d = d;
  qa.m = cf.qjl_bits;
  qa.b_theta = cf.b_theta;
  // q-prep's outputs feed only the cold logits; a gated call always runs it
  // (its gate is q-prep's programmatic dependent)
  if ((pl.cold_ctas > 0 || gate) && launch_qprep(qa, stream) != cudaSuccess) return TQ_ERR_CUDA;
  if (gate) {
    GateArgs ga{};
    ga.q = (const __half*)q;
    ga.hot_k = c->hot_k();
    ga.head_skip = gate->head_skip;
    ga.cmax = gate->cmax;
    ga.unit_pos = gate->unit_pos;
    ga.alist = gate->alist;
    ga.n_active = gate->n_active;
    ga.counter = gate->counter;
    ga.units = units;
    ga.G = cf.num_q_heads / cf.num_kv_heads;
    ga.Hq = cf.num_q_heads;
    ga.Hkv = cf.num_kv_heads;
    ga.W = cf.hot_window;
    ga.n_hot = c->n_hot;
    ga.d = d;
    ga.dirty_lo = c->dirty_lo;
    ga.dirty_n = c->dirty_n;
    ga.threshold = gate->threshold;
    if (launch_gate(ga, stream) != cudaSuccess) return TQ_ERR_CUDA;
  }
  AttendArgs a{};
  a.q = (const __half*)q;
  a.qrot = qb.qrot;
  a.qk8 = qb.qk8;
  a.qs8 = qb.qs8;
  a.qscale = qb.qscale;
  a.hot_k = c->hot_k();
  a.hot_v = c->hot_v();
  a.cold = c->cold;
  a.part = part;
  a.status = c->status();
  a.L = c->L;
  a.units = units;
  a.G = cf.num_q_heads / cf.num_kv_heads;
  a.Hq = cf.num_q_heads;
  a.Hkv = cf.num_kv_heads;
  a.W = cf.hot_window;
  a.n_hot = c->n_hot;
  a.n_cold = c->n_cold;
  a.plan = pl;
  a.rows = rows;
  a.log2e_sigma = (float)(1.4426950408889634 * (double)sigma);
  a.wait_limit_ns = c->wait_limit_ns;
  if (gate) {
    a.alist = gate->alist;
    a.n_active = gate->n_active;
  }
  const bool promo = c->promo != nullptr && gate == nullptr;
  PromoArgs pa{};
  if (promo) {
    pa = promo_args(c);
    a.logits = const_cast<float*>(pa.logits);
    a.logit_capacity = cf.cold_capacity;
  }
  if (c->ev_start && cudaEventRecord(c->ev_start, stream) != cudaSuccess) return TQ_ERR_CUDA;
  if (launch_attend(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  if (c->ev_stop && cudaEventRecord(c->ev_stop, stream) != cudaSuccess) return TQ_ERR_CUDA;
  CombineArgs ca{};
  ca.part = part;
  ca.status = c->status();
  ca.signs = c->signs();
  ca.out = out;
  ca.units = units;
  ca.G = a.G;
  ca.Hkv = cf.num_kv_heads;
  ca.Hq = cf.num_q_heads;
  ca.d = d;
  ca.plan = pl;
  ca.rows = rows;
  ca.batch = cf.batch;
  if (gate) {
    ca.head_skip = gate->head_skip;
    ca.unit_pos = gate->unit_pos;
    ca.n_active = gate->n_active;
  }
  if (promo) ca.ml = const_cast<float*>(pa.ml);
  if (launch_combine(ca, stream) != cudaSuccess) return TQ_ERR_CUDA;
  if (promo && pl.cold_ctas > 0 && launch_promo_mass(pa, stream) != cudaSuccess) return TQ_ERR_CUDA;
  if (c->tc) {
    TcReadArgs tr{};
    tr.A = c->tc;
    tr.sig = c->tc_sig;
    tr.q = (const __half*)q;
    tr.out = out;
    tr.units = units;
    tr.G = a.G;
    tr.Hq = cf.num_q_heads;
    tr.d = d;
    if (launch_tc_read(tr, stream) != cudaSuccess) return TQ_ERR_CUDA;
  }
  return TQ_OK;
}

tq_status tq_decode_attention(tq_cache* c, const void* q, float* out, float softmax_scale,
                              cudaStream_t stream) {
  if (!c || !q || !out || !(softmax_scale >= 0.0f) || std::isinf(softmax_scale) ||
      (uintptr_t)q % 16)
    return TQ_ERR_INVALID_ARG;
  const int units = c->cfg.batch * c->cfg.num_kv_heads;
  if (c->ragged) {
    RowTable t;
    if (upload_rows(c, nullptr, stream, &t) != TQ_OK) return TQ_ERR_CUDA;
    const SplitPlan pl = make_plan_ragged(t, c->cfg.batch, c->cfg.num_kv_heads,
                                          c->num_sms * c->ctas_per_sm, false);
    return launch_decode(c, q, out, softmax_scale, pl, qbufs_at(c->ws + c->W.q, c->W.ql),
                         (float*)(c->ws + c->W.part), stream, nullptr, (const RowTable*)(c->ws + c->W.rows));
  }
  const SplitPlan pl = make_plan(c->n_cold, c->n_hot, units, c->num_sms * c->ctas_per_sm, false);
  return launch_decode(c, q, out, softmax_scale, pl, qbufs_at(c->ws + c->W.q, c->W.ql),
                       (float*)(c->ws + c->W.part), stream);
}

tq_status tq_decode_attention_gated(tq_cache* c, const void* q, float* out, float softmax_scale,
                                    float threshold, int32_t* head_skip, cudaStream_t stream) {
  if (!c || !q || !out || !(softmax_scale >= 0.0f) || std::isinf(softmax_scale) ||
      std::isnan(threshold) || (uintptr_t)q % 16)
    return TQ_ERR_INVALID_ARG;
  if (c->promo || c->ragged) return TQ_ERR_UNSUPPORTED;   // uniform batches, no promotion
  const tq_config& cf = c->cfg;
  const int units = cf.batch * cf.num_kv_heads;
  const int heads = cf.batch * cf.num_q_heads;
  int* area = (int*)(c->ws + c->W.gate);
  GateBuffers gb{};
  gb.head_skip = head_skip ? (int*)head_skip : area;
  gb.cmax = (float*)(c->ws + c->W.gate_max);
  gb.unit_pos = area + heads;
  gb.alist = gb.unit_pos + units;
  gb.n_active = gb.alist + units + 1;
  gb.counter = (unsigned*)(c->ws + c->W.status + 64);   // zeroed at create, reset by each gate
  gb.threshold = threshold;
  const SplitPlan pl = make_plan(c->n_cold, c->n_hot, units, c->num_sms * c->ctas_per_sm, false);
  if (pl.cold_ctas == 0 && pl.hot_ctas == 0 &&        // nothing cached: no head skips
      cudaMemsetAsync(gb.head_skip, 0, sizeof(int) * heads, stream) != cudaSuccess)
    return TQ_ERR_CUDA;
  return launch_decode(c, q, out, softmax_scale, pl, qbufs_at(c->ws + c->W.q, c->W.ql),
                       (float*)(c->ws + c->W.part), stream, &gb);
}

static size_t tc_matrix_bytes(const tq_config& c) {
  return round_up(sizeof(float) * c.batch * c.num_kv_heads * c.head_dim * c.head_dim, kAlign);
}

tq_status tq_tc_bytes(const tq_config* cfg, size_t* bytes) {
  if (!cfg || !bytes) return TQ_ERR_INVALID_ARG;
  const tq_status st = check_config(cfg);
  if (st != TQ_OK) return st;
  *bytes = tc_matrix_bytes(*cfg) +
           round_up(sizeof(float) * (2 * cfg->num_kv_heads + cfg->num_q_heads), kAlign);
  return TQ_OK;
}

tq_status tq_tc_enable(tq_cache* c, void* tc_mem, const float* lambda, const float* eta,
                       const float* gate, cudaStream_t stream) {
  if (!c || !tc_mem || !lambda || !eta || !gate || (uintptr_t)tc_mem % kAlign) return TQ_ERR_INVALID_ARG;
  if (c->tc || c->promo) return TQ_ERR_INVALID_ARG;         // already enabled, or promotion on
  if (c->ragged) return TQ_ERR_UNSUPPORTED;
  const tq_config& cf = c->cfg;
  const int hkv = cf.num_kv_heads, hq = cf.num_q_heads;
  std::vector<float> par(2 * hkv + hq);
  for (int h = 0; h < hkv; ++h) {
    if (!std::isfinite(lambda[h]) || !std::isfinite(eta[h])) return TQ_ERR_INVALID_ARG;
    par[h] = lambda[h];
    par[hkv + h] = eta[h];
  }
  for (int h = 0; h < hq; ++h) {
    if (std::isnan(gate[h])) return TQ_ERR_INVALID_ARG;
    const double g = gate[h];                              // logistic sigmoid without overflow
    par[2 * hkv + h] = (float)(g >= 0 ? 1.0 / (1.0 + std::exp(-g)) : std::exp(g) / (1.0 + std::exp(g)));
  }
  float* A = (float*)tc_mem;
  float* p = (float*)((uint8_t*)tc_mem + tc_matrix_bytes(cf));
  cudaError_t e = cudaMemsetAsync(A, 0, tc_matrix_bytes(cf), stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(p, par.data(), sizeof(float) * par.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);   // `par` is released on return
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  c->tc = A;
  c->tc_lam = p;
  c->tc_eta = p + hkv;
  c->tc_sig = p + 2 * hkv;
  return TQ_OK;
}

tq_status tq_promotion_bytes(const tq_config* cfg, size_t* bytes) {
  if (!cfg || !bytes) return TQ_ERR_INVALID_ARG;
  const tq_status st = check_config(cfg);
  if (st != TQ_OK) return st;
  *bytes = promo_layout(*cfg).total;
  return TQ_OK;
}

tq_status tq_promotion_enable(tq_cache* c, void* mem, float threshold, int32_t sticky,
                              cudaStream_t stream) {
  if (!c || !mem || (uintptr_t)mem % kAlign || !(threshold >= 0.125f && threshold <= 1.0f) ||
      sticky < 1 || c->cfg.hot_window <= kPromoMax)
    return TQ_ERR_INVALID_ARG;
  if (c->tc || c->promo) return TQ_ERR_INVALID_ARG;        // Tensor Cache tier, or already on
  if (c->ragged) return TQ_ERR_UNSUPPORTED;
  const size_t units = (size_t)c->cfg.batch * c->cfg.num_kv_heads;
  std::vector<PromoUnitState> st(units);
  for (auto& u : st) {
    for (int i = 0; i < kPromoMax; ++i) {
      u.cnt_idx[i] = -1;
      u.cnt_val[i] = 0;
      u.pend_idx[i] = -1;
    }
    u.n_cnt = u.n_pend = 0;
    u.ring_pos = c->ring_pos;
    for (int& x : u.pad) x = 0;
  }
  cudaError_t e = cudaMemcpyAsync(mem, st.data(), sizeof(PromoUnitState) * units, cudaMemcpyHostToDevice,
                                  stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);   // `st` is released on return
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  c->promo = (uint8_t*)mem;
  c->promo_threshold = threshold;
  c->promo_sticky = sticky;
  return TQ_OK;
}

tq_status tq_promotion_state(tq_cache* c, int32_t* out, cudaStream_t stream) {
  if (!c || !out) return TQ_ERR_INVALID_ARG;
  if (!c->promo) return TQ_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  const size_t units = (size_t)c->cfg.batch * c->cfg.num_kv_heads;
  std::vector<PromoUnitState> st(units);
  if (cudaMemcpy(st.data(), c->promo + promo_layout(c->cfg).state, sizeof(PromoUnitState) * units,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return TQ_ERR_CUDA;
  for (size_t u = 0; u < units; ++u) {
    int32_t* o = out + u * 28;
    o[0] = st[u].n_cnt;
    o[1] = st[u].n_pend;
    o[2] = st[u].ring_pos;
    o[3] = 0;
    for (int i = 0; i < kPromoMax; ++i) {
      o[4 + i] = st[u].cnt_idx[i];
      o[12 + i] = st[u].cnt_val[i];
      o[20 + i] = st[u].pend_idx[i];
    }
  }
  return TQ_OK;
}

tq_status tq_set_wait_limit(tq_cache* c, int64_t limit_ns) {
  if (!c) return TQ_ERR_INVALID_ARG;
  c->wait_limit_ns = limit_ns < 0 ? kDefaultWaitLimitNs : (unsigned long long)limit_ns;
  return TQ_OK;
}

tq_status tq_set_attend_events(tq_cache* c, cudaEvent_t start, cudaEvent_t stop) {
  if (!c || (start == nullptr) != (stop == nullptr)) return TQ_ERR_INVALID_ARG;
  c->ev_start = start;
  c->ev_stop = stop;
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// Decode attention with library-owned static scratch.
//
// Some callers may not allocate device memory while they run: code inside
// an allocator-free serving loop, a plugin whose host framework owns every
// allocation, or a process whose memory is fully reserved up front.  For
// them tq_decode_attention_static keeps the per-call scratch (the rotated
// queries and the split partials) in one fixed device array compiled into
// this library instead of the handle's workspace.  The array exists once
// per GPU that loads the library and stays resident until the process
// exits.  Calls that overlap on the GPU share it and race; nothing in it has
// to start at zero, because every call writes what it reads.
// ---------------------------------------------------------------------------
static constexpr size_t kStaticScratchBytes = (size_t)4 << 20;   // 4 MiB
static __device__ __align__(256) unsigned char tq_static_scratch[kStaticScratchBytes];

static constexpr int kMaxScratchDevices = 64;
static std::mutex g_static_scratch_mu;
static void* g_static_scratch_ptr[kMaxScratchDevices] = {};

// Device address of tq_static_scratch on `device`, which must be current.
// The name is only a host-side stand-in: the address is fetched once per
// device with cudaGetSymbolAddress and remembered.
static void* static_scratch_address(int device) {
  if (device < 0 || device >= kMaxScratchDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_ptr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, tq_static_scratch) != cudaSuccess || !p) return nullptr;
    g_static_scratch_ptr[device] = p;
  }
  return g_static_scratch_ptr[device];
}

tq_status tq_decode_attention_static(tq_cache* c, const void* q, float* out, float softmax_scale,
                                     cudaStream_t stream) {
  if (!c || !q || !out || !(softmax_scale >= 0.0f) || std::isinf(softmax_scale) ||
      (uintptr_t)q % 16)
    return TQ_ERR_INVALID_ARG;
  int current = -1;
  if (cudaGetDevice(&current) != cudaSuccess) return TQ_ERR_CUDA;
  if (current != c->device) return TQ_ERR_INVALID_ARG;   // the handle's GPU must be current
  const tq_config& cf = c->cfg;
  const int d = cf.head_dim, m = cf.qjl_bits;
  const int heads = cf.batch * cf.num_q_heads;
  const int units = cf.batch * cf.num_kv_heads;
  const int G = cf.num_q_heads / cf.num_kv_heads;

  // The same split plan as tq_decode_attention, with the partial slots per
  // unit cut to the most any unit can receive under this plan.
  RowTable t{};
  if (c->ragged) t = build_rows(c, nullptr);    // (a ragged batch has at most kMaxRaggedRows rows)
  const SplitPlan pl = c->ragged ? make_plan_ragged(t, cf.batch, cf.num_kv_heads, c->num_sms * c->ctas_per_sm, true)
                                 : make_plan(c->n_cold, c->n_hot, units, c->num_sms * c->ctas_per_sm, true);

  // scratch layout: query transforms | partials
  const QBufsLayout ql = qbufs_layout((size_t)heads, d, m);
  size_t off = ql.total;
  const size_t o_part = off;
  off += round_up(sizeof(float) * units * (size_t)(pl.slots_cold + pl.slots_hot) * G * (d + 2), kAlign);
  if (off > kStaticScratchBytes) return TQ_ERR_CAPACITY;   // too large for the static scratch

  uint8_t* base = (uint8_t*)static_scratch_address(current);
  if (!base) return TQ_ERR_CUDA;
  if (c->ragged && launch_rows_upload((RowTable*)(c->ws + c->W.rows), t, stream) != cudaSuccess)
    return TQ_ERR_CUDA;
  return launch_decode(c, q, out, softmax_scale, pl, qbufs_at(base, ql), (float*)(base + o_part), stream,
                       nullptr, c->ragged ? (const RowTable*)(c->ws + c->W.rows) : nullptr);
}

tq_status tq_get_status(tq_cache* c, cudaStream_t stream) {
  if (!c) return TQ_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, c->status(), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (word != 0 && cudaMemset(c->status(), 0, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  if (word & kStatusLayout) return TQ_ERR_UNSUPPORTED;
  if (word & kStatusTimeout) return TQ_ERR_TIMEOUT;
  if (word & kStatusRange) return TQ_ERR_RANGE;
  return TQ_OK;
}

tq_status tq_export_cold(tq_cache* c, int32_t row, int32_t kv_head, int64_t start, int64_t count,
                         uint8_t* k_codes, uint8_t* k_bits, uint16_t* k_s16, uint16_t* k_rn16,
                         uint8_t* v_codes, uint16_t* v_s16, cudaStream_t stream) {
  if (!c || row < 0 || row >= c->cfg.batch || kv_head < 0 || kv_head >= c->cfg.num_kv_heads ||
      start < 0 || count < 0 || start + count > c->row_cold[row])
    return TQ_ERR_INVALID_ARG;
  if (count == 0) return TQ_OK;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  const Layout& L = c->L;
  const int TB = kTokensPerBlock;
  const int64_t unit = (int64_t)row * c->cfg.num_kv_heads + kv_head;
  const int64_t b0 = start / TB, b1 = (start + count - 1) / TB;
  std::vector<uint8_t> buf((size_t)(b1 - b0 + 1) * L.block_bytes);
  const uint8_t* src = c->cold + ((size_t)unit * L.blocks_per_unit + b0) * L.block_bytes;
  if (cudaMemcpy(buf.data(), src, buf.size(), cudaMemcpyDeviceToHost) != cudaSuccess)
    return TQ_ERR_CUDA;
  const int bw = L.bw;
  auto word_at = [&](const uint8_t* plane, int w, int lane, int nw) {
    uint32_t v;
    std::memcpy(&v, plane + lane_word_offset(w, lane, nw), 4);
    return v;
  };
  // bit `bit` of a lane chunk stream of nw words
  auto chunk_bits = [&](const uint8_t* plane, int lane, int nw, int bit, int width) {
    const int w = bit >> 5, sh = bit & 31;
    uint64_t v = word_at(plane, w, lane, nw);
    if (sh + width > 32 && w + 1 < nw) v |= (uint64_t)word_at(plane, w + 1, lane, nw) << 32;
    return (uint32_t)((v >> sh) & ((1ull << width) - 1));
  };
  auto put_bits = [](uint8_t* out, int bit, uint32_t val, int width) {
    for (int b = 0; b < width; ++b)
      if ((val >> b) & 1u) out[(bit + b) >> 3] |= (uint8_t)(1u << ((bit + b) & 7));
  };
  for (int64_t i = 0; i < count; ++i) {
    const int64_t t = start + i;
    const uint8_t* blk = buf.data() + (size_t)(t / TB - b0) * L.block_bytes;
    const int tok = (int)(t % TB);
    const uint8_t* tile = blk + (tok / kTokensPerTile) * L.tile_bytes;
    const int r = tok % kTokensPerTile;
    const int gid = r % 8, h = r / 8;
    if (k_codes) {
      uint8_t* out = k_codes + i * L.kc_bytes;
      std::memset(out, 0, L.kc_bytes);
      for (int p = 0; p < L.pairs; ++p) {
        const int tig = p / L.pt, k = p % L.pt;
        put_bits(out, p * bw, chunk_bits(tile + L.off_kc, 4 * gid + tig, L.kwt, (h * L.pt + k) * bw, bw), bw);
      }
    }
    if (v_codes) {
      uint8_t* out = v_codes + i * L.kc_bytes;
      std::memset(out, 0, L.kc_bytes);
      for (int p = 0; p < L.pairs; ++p) {
        const int tig = p / L.pt, k = p % L.pt;
        put_bits(out, p * bw, chunk_bits(tile + L.off_vc, 4 * gid + tig, L.vwt, (h * L.pt + k) * bw, bw), bw);
      }
    }
    if (k_bits) {
      uint8_t* out = k_bits + i * L.sg_bytes;
      std::memset(out, 0, L.sg_bytes);
      const int qb = L.m / 4;
      for (int tig = 0; tig < 4; ++tig)
        for (int j = 0; j < qb; ++j)
          put_bits(out, tig * qb + j, chunk_bits(tile + L.off_ks, 4 * gid + tig, L.sw,
                                                 sign_chunk_bit(j, h, L.m), 1), 1);
    }
    const uint16_t* ks = reinterpret_cast<const uint16_t*>(tile + L.off_ksc);
    const uint16_t* vs = reinterpret_cast<const uint16_t*>(tile + L.off_vsc);
    if (k_s16) k_s16[i] = ks[gid * 4 + h];
    if (k_rn16) k_rn16[i] = ks[gid * 4 + 2 + h];
    if (v_s16) v_s16[i] = vs[gid * 2 + h];
  }
  return TQ_OK;
}

tq_status tq_rotation_signs(uint64_t seed, int32_t d, int8_t* signs) {
  if (!signs || d < 1) return TQ_ERR_INVALID_ARG;
  std::vector<double> s(d);
  gen_signs(seed, d, s.data());
  for (int i = 0; i < d; ++i) signs[i] = (int8_t)s[i];
  return TQ_OK;
}

tq_status tq_qjl_matrix(uint64_t seed, int32_t m, int32_t d, float* S) {
  if (!S || m < 1 || d < 1) return TQ_ERR_INVALID_ARG;
  gen_qjl(seed, m, d, S);
  return TQ_OK;
}

}  // extern "C"
