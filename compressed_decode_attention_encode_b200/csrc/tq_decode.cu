// Decode attention straight from the packed cold cache plus the fp16 hot
// ring ("TurboQuant: optimización de memoria para KV caches en inferencia
// de LLMs", flow step 6: attention logits from the compressed cache;
// "Monarch v3 ...", "Bucle de Decodificación Simplificado": aggregate the hot
// and cold scores, softmax, apply).
//
// Three launches per call:
//   qprep    q' = R q (fp32 Hadamard butterflies), q'' = S q', and their
//            tensor-core operands: q' as fp16 hi + lo parts, the
//            projections of q' on the polar slot directions and q'' as two
//            int8 planes each, with their scales.
//   attend   the attention kernel (tq_attend.cuh, instantiated per shape in
//            tq_attend_<d>_<m>.cu): split partials over hot and cold tokens.
//   combine  merges the partials of each (row, head), applies R^T once to
//            the cold sum (Hadamard butterflies) and normalizes.
// A gated call (tq_decode_attention_gated) runs the gate of tq_gate.cu
// between qprep and attend; its attention kernel streams the cold blocks of
// the listed units only, split again over the same CTAs, and combine leaves
// out the cold partials of the heads that skipped.
#include <cfloat>

#include "tq_attend.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kNegInf = -INFINITY;
constexpr int kPlaneMax = 127 * 256 + 127;   // largest |x| of two int8 planes x = 256 hi + lo

// x (|x| <= kPlaneMax) as planes hi, lo in [-128, 127]: x = 256 hi + lo.
__device__ __forceinline__ void split_planes(int x, int8_t* hi, int8_t* lo) {
  const int h = (x + 128) >> 8;            // floor((x + 128) / 256)
  *hi = (int8_t)h;
  *lo = (int8_t)(x - 256 * h);
}

// Integer value of v in units of alpha = amax / kPlaneMax, clamped.
__device__ __forceinline__ int to_units(float v, float inv_alpha) {
  int x = __float2int_rn(v * inv_alpha);
  return x > kPlaneMax ? kPlaneMax : (x < -kPlaneMax ? -kPlaneMax : x);
}

// ---------------------------------------------------------------------------
// q-prep: HB = 256 / M heads per block (2 for m = 128), so that the grid
// spreads over the SMs.  One warp per head rotates q (butterflies in
// registers and across lanes) and writes q' as fp16 hi + lo and the int8
// planes of its slot projections; then every thread computes one element
// of S q' from S^T staged in shared memory (asynchronous copies issued
// before the rotation), and the head's warp writes the planes of q''.
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
  constexpr int PT = D / 8;              // pairs per B-fragment lane group
  constexpr int NT = D / 16;             // K k-steps
  constexpr int QB = M / 4;              // signs per B-fragment lane group
  constexpr int QS = M / 32;             // QJL k-steps
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
    // projections of the lane's pairs on the slot directions e(pi k / ns)
    const int bt = a.b_theta;
    const int ns = bt <= 1 ? 1 : (bt == 2 ? 2 : 4);
    float pr[E / 2][4];
    float pmax = 0.f;
#pragma unroll
    for (int k = 0; k < E / 2; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float sn, cs;
        sincospif((float)e / (float)ns, &sn, &cs);
        pr[k][e] = e < ns ? fmaf(x[2 * k], cs, x[2 * k + 1] * sn) : 0.f;
        pmax = fmaxf(pmax, fabsf(pr[k][e]));
      }
#pragma unroll
    for (int o = 16; o; o >>= 1) pmax = fmaxf(pmax, __shfl_xor_sync(kFull, pmax, o));
    if (live) {
      __half* qrot = a.out.qrot + (size_t)h * 2 * D;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float v = x[i] * al1;
        const __half hi = __float2half_rn(v);
        qrot[lane * E + i] = hi;
        qrot[D + lane * E + i] = __float2half_rn(v - __half2float(hi));
      }
      const float inv_ak = pmax > 0.f ? (float)kPlaneMax / pmax : 0.f;
      int8_t* qk = a.out.qk8 + (size_t)h * 2 * NT * 32;
#pragma unroll
      for (int k = 0; k < E / 2; ++k) {
        const int p = lane * (E / 2) + k;
        const int t = p / PT, kk = p % PT;
        const int off = (kk >> 1) * 32 + t * 8 + 4 * (kk & 1);
#pragma unroll
        for (int e = 0; e < 4; ++e) split_planes(to_units(pr[k][e], inv_ak), qk + off + e, qk + NT * 32 + off + e);
      }
      if (lane == 0) {
        a.out.qscale[4 * h + 0] = 1.f / al1;
        a.out.qscale[4 * h + 1] = pmax > 0.f ? pmax / (float)kPlaneMax : 0.f;
      }
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
  const float inv_as = bmax > 0.f ? (float)kPlaneMax / bmax : 0.f;
  int8_t* qs = a.out.qs8 + (size_t)h * 2 * QS * 32;
  int sum = 0;
  for (int i = lane; i < M; i += 32) {
    const int x = to_units(sqq[warp][i], inv_as);
    sum += x;
    const int t = i / QB, j = i % QB;
    const int off = (j >> 3) * 32 + t * 8 + 4 * ((j >> 2) & 1) + (j & 3);
    split_planes(x, qs + off, qs + QS * 32 + off);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
  if (lane == 0) {
    a.out.qscale[4 * h + 2] = bmax > 0.f ? bmax / (float)kPlaneMax : 0.f;
    a.out.qscale[4 * h + 3] = __int_as_float(sum);
  }
}

// ---------------------------------------------------------------------------
// combine
// ---------------------------------------------------------------------------
// One block per query head; its kCombineWarps warps split the head's slots
// (contiguous quarters), lane i holding output dims [PD i, PD i + PD).  The
// kernel moves a few KB per head and is bound by load latency, so its loads
// go out together: a warp's (m, l) pairs one per lane, the o vectors of up
// to kCombineChunk of its slots before anything waits on a load.  Each warp
// merges its slots against its own max; the warps' (m, l, o) are then
// rescaled to the head's max and added in warp order through shared memory,
// and warp 0 applies R^T to the cold sum with butterflies inside the lane
// and across lanes (shuffles).
constexpr int kCombineMaxSlots = kSlotsCold + kSlotsHot;
constexpr int kCombineChunk = 16;    // slots whose o vectors are in flight together
constexpr int kCombineWarps = 4;     // warps per head (slots per warp <= 32)
static_assert(kCombineMaxSlots <= 32 * kCombineWarps, "one (m, l) pair per lane");

template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const CombineArgs a) {
  constexpr int PD = D / 32;
  constexpr int CH = kCombineChunk;
  constexpr int NW = kCombineWarps;
  __shared__ float s_ml[NW][2];
  __shared__ float s_o[NW][2][D];
  // The next step's eviction encode may start its prologue now (it waits
  // for this kernel before reading its inputs).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // launched as a programmatic dependent of the attention kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hg = blockIdx.x;
  const int b = hg / a.Hq, hq = hg % a.Hq;
  const int kvh = hq / a.G, g = hq % a.G;
  const int unit = b * a.Hkv + kvh;
  const SplitPlan& pl = a.plan;
  const int slots = pl.slots_cold + pl.slots_hot;
  const float* base = a.part + (size_t)unit * slots * a.G * (D + 2);
  int nc = 0, nh = 0;
  if (a.rows != nullptr) {             // ragged: the unit's own blocks and tiles
    const int h = unit % a.Hkv;
    const int64_t nb = (a.rows->n_cold[b] + kTokensPerBlock - 1) / kTokensPerBlock;
    const int64_t ht = (a.rows->n_hot[b] + kTokensPerBlock - 1) / kTokensPerBlock;
    if (nb > 0) {
      const int64_t off = a.rows->cold_pre[b] + h * nb;
      nc = (int)((off + nb - 1) / pl.cold_bpc - off / pl.cold_bpc + 1);
    }
    if (ht > 0) {
      const int64_t off = a.rows->hot_pre[b] + h * ht;
      nh = (int)((off + ht - 1) / pl.hot_tpc - off / pl.hot_tpc + 1);
    }
  } else if (pl.cold_ctas > 0 && pl.cold_blocks > 0) {
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
  if (a.rows == nullptr && pl.hot_ctas > 0 && pl.hot_tiles > 0) {
    const int64_t ht = pl.hot_tiles;
    nh = (int)(((unit + 1) * ht - 1) / pl.hot_tpc - (unit * ht) / pl.hot_tpc + 1);
  }
  const int ns = nc + nh;
  auto rec = [&](int s) {
    return base + ((size_t)(s < nc ? s : pl.slots_cold + (s - nc)) * a.G + g) * (D + 2);
  };
  // this lane's dims of slot s's o vector (records are 8-byte aligned)
  auto load_o = [&](int s, float (&o)[PD]) {
    const float* pp = rec(s) + 2 + lane * PD;
#pragma unroll
    for (int k = 0; k < PD; k += 2) {
      const float2 v = *reinterpret_cast<const float2*>(pp + k);
      o[k] = v.x;
      o[k + 1] = v.y;
    }
  };
  const int lo = warp * ns / NW, hi = (warp + 1) * ns / NW;   // this warp's slots
  float ov[CH][PD];
#pragma unroll
  for (int u = 0; u < CH; ++u) {
    if (lo + u < hi) {
      load_o(lo + u, ov[u]);
    } else {
#pragma unroll
      for (int k = 0; k < PD; ++k) ov[u][k] = 0.f;
    }
  }
  float ms = kNegInf, ls = 0.f;              // slot lo + lane
  if (lo + lane < hi) {
    const float2 v = *reinterpret_cast<const float2*>(rec(lo + lane));
    ms = v.x;
    ls = v.y;
  }
  float* orow = a.out + (size_t)hg * D + lane * PD;
  if (*(volatile const int*)a.status & kStatusNoPartials) {
    // an attention launch gave up without writing its partials (a latched
    // timeout or layout error): the output is NaN until the status is read
    if (warp == 0)
#pragma unroll
      for (int k = 0; k < PD; ++k) orow[k] = __int_as_float(0x7fc00000);
    return;
  }
  // ---- this warp: m_w = max over its slots, w_s = 2^(m_s - m_w), l_w -------
  float mw = ms;
#pragma unroll
  for (int o = 16; o; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(kFull, mw, o));
  const float ws = ms == kNegInf ? 0.f : exp2f(ms - mw);
  float lw = ws * ls;
#pragma unroll
  for (int o = 16; o; o >>= 1) lw += __shfl_xor_sync(kFull, lw, o);
  float oc[PD], oh[PD];
#pragma unroll
  for (int k = 0; k < PD; ++k) oc[k] = oh[k] = 0.f;
  auto accum = [&](int s, const float (&o)[PD]) {   // (s warp-uniform)
    const float wt = __shfl_sync(kFull, ws, s - lo);
    if (s < nc) {
#pragma unroll
      for (int k = 0; k < PD; ++k) oc[k] += wt * o[k];
    } else {
#pragma unroll
      for (int k = 0; k < PD; ++k) oh[k] += wt * o[k];
    }
  };
  if (mw != kNegInf) {
#pragma unroll
    for (int u = 0; u < CH; ++u)
      if (lo + u < hi) accum(lo + u, ov[u]);
    for (int s0 = lo + CH; s0 < hi; s0 += CH) {
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (s0 + u < hi) load_o(s0 + u, ov[u]);
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (s0 + u < hi) accum(s0 + u, ov[u]);
    }
  }
  if (lane == 0) {
    s_ml[warp][0] = mw;
    s_ml[warp][1] = lw;
  }
#pragma unroll
  for (int k = 0; k < PD; ++k) {
    s_o[warp][0][lane * PD + k] = oc[k];
    s_o[warp][1][lane * PD + k] = oh[k];
  }
  __syncthreads();
  if (warp != 0) return;
  // ---- the head: m = max of the warps' maxima; each warp's sums scaled by
  // 2^(m_w - m) and added in warp order ------------------------------------
  float mx = s_ml[0][0];
#pragma unroll
  for (int w = 1; w < NW; ++w) mx = fmaxf(mx, s_ml[w][0]);
  float lsum = 0.f;
#pragma unroll
  for (int k = 0; k < PD; ++k) oc[k] = oh[k] = 0.f;
  if (mx != kNegInf) {
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = s_ml[w][0] == kNegInf ? 0.f : exp2f(s_ml[w][0] - mx);
      lsum += f * s_ml[w][1];
#pragma unroll
      for (int k = 0; k < PD; ++k) {
        oc[k] += f * s_o[w][0][lane * PD + k];
        oh[k] += f * s_o[w][1][lane * PD + k];
      }
    }
  }
  // ---- R^T on the cold sum: unnormalised Hadamard (dim i = PD lane + k),
  // strides below PD inside the lane, the others across lanes; then the
  // signs and 1/sqrt(d) ----------------------------------------------------------
#pragma unroll
  for (int h = 1; h < PD; h <<= 1)
#pragma unroll
    for (int k = 0; k < PD; ++k)
      if (!(k & h)) {
        const float x = oc[k], y = oc[k + h];
        oc[k] = x + y;
        oc[k + h] = x - y;
      }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int k = 0; k < PD; ++k) {
      const float o = __shfl_xor_sync(kFull, oc[k], h);
      oc[k] = (lane & h) ? (o - oc[k]) : (oc[k] + o);
    }
  const float rs = rsqrtf((float)D);
#pragma unroll
  for (int k = 0; k < PD; ++k)
    orow[k] = mx == kNegInf ? 0.f : (oh[k] + (float)a.signs[lane * PD + k] * oc[k] * rs) / lsum;
  if (a.ml != nullptr && lane == 0) {   // the softmax's normaliser, for promotion
    a.ml[2 * (size_t)hg] = mx;
    a.ml[2 * (size_t)hg + 1] = lsum;
  }
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
att::AttendFn pick_attend(const Layout& L, int G, int mode, int* smem) {
  if (L.d == 64 && L.m == 64) return attend_pick_64_64(L.bw, L.b_theta, G, mode, smem);
  if (L.d == 64 && L.m == 128) return attend_pick_64_128(L.bw, L.b_theta, G, mode, smem);
  if (L.d == 128 && L.m == 64) return attend_pick_128_64(L.bw, L.b_theta, G, mode, smem);
  if (L.d == 128 && L.m == 128) return attend_pick_128_128(L.bw, L.b_theta, G, mode, smem);
  return nullptr;
}

}  // namespace

int attend_ctas_per_sm(const Layout& L, int G) {
  int smem = 0, n = 0;
  for (int mode = att::MODE_PLAIN; mode <= att::MODE_RAGGED; ++mode) {
    att::AttendFn fn = pick_attend(L, G, mode, &smem);
    if (!fn || cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return 0;
    if (mode == att::MODE_PLAIN &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, att::kThreads, smem) != cudaSuccess)
      return 0;
  }
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
  const int mode = a.alist ? att::MODE_GATED
                 : a.logits ? att::MODE_LOGITS
                 : a.rows ? att::MODE_RAGGED : att::MODE_PLAIN;
  att::AttendFn fn = pick_attend(a.L, a.G, mode, &smem);
  if (!fn) return cudaErrorInvalidValue;
  const int grid = a.plan.cold_ctas > a.plan.hot_ctas ? a.plan.cold_ctas : a.plan.hot_ctas;
  if (grid == 0) return cudaSuccess;
  fn<<<grid, att::kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

namespace {
__global__ void rows_upload_kernel(RowTable* dst, const RowTable src) {
  const int32_t* s = reinterpret_cast<const int32_t*>(&src);
  int32_t* d = reinterpret_cast<int32_t*>(dst);
  for (int i = threadIdx.x; i < (int)(sizeof(RowTable) / 4); i += blockDim.x) d[i] = s[i];
}
}  // namespace

cudaError_t launch_rows_upload(RowTable* dst, const RowTable& src, cudaStream_t s) {
  rows_upload_kernel<<<1, 256, 0, s>>>(dst, src);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  if (a.d != 64 && a.d != 128) return cudaErrorInvalidValue;
  // programmatic dependent launch: the kernel waits for the attention
  // kernel before it reads the partials
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.batch * a.Hq);
  cfg.blockDim = dim3(32 * kCombineWarps);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.d == 64) return cudaLaunchKernelEx(&cfg, combine_kernel<64>, a);
  return cudaLaunchKernelEx(&cfg, combine_kernel<128>, a);
}

}  // namespace tq
