// Internal declarations shared by the library's CUDA translation units.
// Layout of the packed cold store, kernel argument blocks and launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/tq.h"

namespace tq {

// Tokens per cold block.  A block holds field planes, each token-major:
//   K codes [TB][kc_bytes] | K signs [TB][sg_bytes] | K s16 [TB] | K rn16 [TB]
//   | V codes [TB][kc_bytes] | V s16 [TB]
// With TB = 64 every plane starts on a 16-byte boundary.
constexpr int kTokensPerBlock = 64;

// Device status word bits (latched, cleared by tq_get_status).
constexpr int kStatusRange = 1;
constexpr int kStatusTimeout = 2;

struct Layout {
  int d;            // head_dim (power of two)
  int pairs;        // d / 2
  int b_r, b_theta, bw;
  int m;            // QJL bits
  int kc_bytes;     // packed code bytes per vector: pairs * bw / 8
  int sg_bytes;     // m / 8
  // plane offsets inside a block
  int off_kc, off_ks, off_ksc, off_krn, off_vc, off_vsc;
  int block_bytes;
  int64_t blocks_per_unit;  // ceil(cold_capacity / TB)
};

Layout make_layout(int d, int b_r, int b_theta, int m, int64_t capacity);

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
  int* status;
  double inv_sqrt_d;        // 1 / sqrt(d), correctly rounded on the host
};

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s);

// Copies new tokens i in [first, n) into ring slots (ring_pos + i) mod W.
cudaError_t launch_ring_write(__half* ring_k, __half* ring_v, const __half* k_new,
                              const __half* v_new, int units, int W, int d, int n,
                              int first, int ring_pos, cudaStream_t s);

// ---- decode -------------------------------------------------------------
struct QPrepArgs {
  const __half* q;          // [B*Hq, d]
  const double* signs;      // [d]
  const float* St;          // [d, m]
  __half* qrot;             // [B*Hq, d]   q' * alpha'
  __half* qsk;              // [B*Hq, m]   q'' * alpha'' in sign-fragment order
  float* qscale;            // [B*Hq, 2]   1/alpha', 1/alpha''
  int heads;                // B*Hq
  int d, m;
};

cudaError_t launch_qprep(const QPrepArgs& a, cudaStream_t s);

struct Partial;  // per (unit, split, head): m (log2 units), l, o[d]

struct AttendArgs {
  const __half* q;          // [B*Hq, d]  (hot logits use q itself)
  const __half* qrot;       // q' fragments source
  const __half* qsk;        // q'' fragments source
  const float* qscale;
  const __half* hot_k;      // [units, W, d]
  const __half* hot_v;
  const uint8_t* cold;
  float* part;              // [units, max_splits, G, d + 2]
  int* status;
  Layout L;
  int units, G, Hq, Hkv;
  int W, n_hot;
  int64_t n_cold;
  int ns_cold, ns_hot;      // splits per unit
  int blocks_per_split;     // cold blocks per cold split
  int tiles_per_split;      // 64-token hot tiles per hot split
  int max_splits;
  float log2e_sigma;        // log2(e) * softmax scale
};

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s);
int attend_ctas_per_sm(const Layout& L);

struct CombineArgs {
  const float* part;
  const double* signs;
  float* out;               // [B*Hq, d]
  int units, G, Hkv, Hq, d, batch;
  int ns_cold, ns_hot, max_splits;
};

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

}  // namespace tq
