// Vector inner-product search over TurboQuant codes ("Compresión del caché
// KV de los LLM a 3 bits: TurboQuant de Google Research", section
// "Aplicaciones más allá de los LLMs": the same compressed vectors rank a
// database for vector search / RAG).
//
//   vec_encode_kernel   float32 vectors -> codes, one warp per vector; the
//                       float64 decision path of the KV encoder.  Records
//                       are stored in groups of 32 vectors, 16-byte chunks
//                       chunk-major, so that a warp reading one chunk of 32
//                       vectors reads 512 contiguous bytes.
//   vec_qprep_kernel    q' = R q, q'' = S q' written as the fp16 A operand of
//                       the search MMAs, one row per query (rows padded to
//                       whole tiles of 128 with zeros).
//   search_umma_kernel  per CTA: 128 queries (A, resident in tensor memory)
//                       against a contiguous run of the database, 128
//                       vectors per round.  Eight producer warps dequantize
//                       the round's vectors straight into the B operand in
//                       shared memory (fp16 c_r (cos, sin) from a LUT times
//                       s16/(2^b_r-1); QJL signs as +-rn16 sqrt(pi/2)/m);
//                       one thread issues tcgen05.mma (M 128, N 128, K 16,
//                       A from tensor memory) into one of two fp32
//                       accumulators; eight epilogue warps read the scores
//                       back (thread = query, one warp group per column
//                       half) and keep each query's 16 best per half.
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
constexpr int kListK = 16;               // best candidates kept per (query, split); k <= kListK
constexpr int kMaxSplits = 32;           // database splits per search (grid y)
constexpr float kNegInf = -INFINITY;

// Search tile shape (tcgen05, one CTA per SM).
constexpr int kM = 128;                  // queries per CTA = MMA M = tensor-memory lanes
constexpr int kN = 128;                  // database vectors per round = MMA N
constexpr int kRingKSteps = 32;          // B ring: 32 k-steps (16 k each) of kN rows
constexpr int kMaxStages = 8;            // stages of the ring: 4 k-steps (d = 64) or 8
constexpr int kQ = 16;                   // candidate queue entries per (query, round parity)
constexpr int kEpiWarps = 8;             // warps 0-7: lane quarter w % 4, column half w / 4
constexpr int kProdWarps = 8;            // warps 8-15: vector 32 (w % 4) + lane, k-step half w / 4
constexpr int kMmaWarp = kEpiWarps + kProdWarps;
constexpr int kSearchThreads = (kMmaWarp + 1) * 32;
constexpr int kKStepB = kN * 32;         // bytes of one B k-step (128 rows x 16 fp16)
constexpr uint32_t kTmemCols = 512;      // accumulators at columns 0 and kN, A from column 2 kN
constexpr uint32_t kTmemA = 2 * kN;
// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), fp16 A and B (bits 7-12 = 0), both K-major (bits 15-16 = 0),
// N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);

// Dynamic shared memory of the search kernel.
struct SearchSmem {
  static constexpr int LUT = 0;                              // 256 entries x 32 lane copies x 4 B
  static constexpr int B = LUT + 256 * 32 * 4;               // the B ring
  static constexpr int QUEUE = B + kRingKSteps * kKStepB;    // [kQ][8 warps x 32] (score, index)
  static constexpr int BAR = QUEUE + kQ * kEpiWarps * 32 * 8;  // full[8], empty[8], acc_full[2], acc_empty[2], done
  static constexpr int TMEM_SLOT = BAR + 8 * (2 * kMaxStages + 5);
  static constexpr int ABORT = TMEM_SLOT + 4;
  static constexpr int BYTES = (ABORT + 4 + 127) / 128 * 128;
};

// QJL k-steps of the search operands for m sign bits.  Sign word w (bits
// 32w..32w+31) fills k-steps 2w and 2w + 1 (half h = 0, 1): in half h,
// chunk kc, half2 u holds bits 15-u' (low half) and 31-u' (high half) of the
// word, u' = 8h + 4kc + u, so one shift and one logic op turn a sign word
// into a B register.  When the last word holds only 8 needed bits
// (m % 32 == 8), they are bits 0-7, all in the low halves of h = 1, and
// h = 0 is skipped.
__host__ __device__ inline int search_qjl_steps(int m) {
  const int r = m % 32;
  return 2 * (m / 32) + (r == 0 ? 0 : (r == 8 ? 1 : 2));
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

// ---- shared memory, barriers, tensor memory ---------------------------------
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void sts64f(uint32_t addr, float x, float y) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}

// Streaming loads straight into the destination registers (nothing reads
// them until a round later, so the loads stay in flight meanwhile).
__device__ __forceinline__ void ldg_stream4(const void* p, uint32_t& x, uint32_t& y, uint32_t& z, uint32_t& w) {
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(x), "=r"(y), "=r"(z), "=r"(w)
               : "l"(p));
}

__device__ __forceinline__ void ldg_stream1(const void* p, uint32_t& x) {
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(x) : "l"(p));
}

__device__ __forceinline__ void ldg_stream_u16(const void* p, uint32_t& x) {
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=r"(x) : "l"(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// try_wait that may suspend the thread (it issues nothing meanwhile) until
// the phase completes or about kSuspendNs have passed.
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_wait_suspend(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of an mbarrier.  Gives up when another role has
// raised the CTA's abort flag, or after `limit_ns` (then raises it and
// latches kStatusTimeout).
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                              volatile int* abort_flag, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_wait_suspend(bar, parity)) {
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// One lane waits, the warp learns the outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                          volatile int* abort_flag, int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, limit_ns, abort_flag, status) ? 1 : 0;
  return __shfl_sync(kFull, ok, 0) != 0;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major, no-swizzle shared-memory matrix descriptor: core matrices of 8
// rows x 16 bytes; the two 8-element K halves of a k-step 128 bytes apart
// (leading byte offset), 8-row groups 256 bytes apart (stride byte offset);
// descriptor version 1 at bit 46.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(256 >> 4) << 32) |
         (1ull << 46);
}

// D (+)= A B^T, kind::f16, A in tensor memory (lane = row, fp16 element k
// of a row in 32-bit column k / 2, even k in the low half), B by descriptor.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The mbarrier's arrival once every tcgen05.mma this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_saddr, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.  The
// wait names the registers so that no use of them moves above it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// ---- the per-query best list -------------------------------------------------
// Inserts (s, v) into a list sorted by (score desc, index asc) whose
// indices are all below v: v goes after every entry scoring >= s.
template <int K>
__device__ __forceinline__ void list_insert(float (&ts)[K], int (&ti)[K], float s, int v) {
  bool pc = false;
  float ps = 0.f;
  int pi = 0;
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const bool c = s > ts[j];
    const float os = ts[j];
    const int oi = ti[j];
    ts[j] = pc ? ps : (c ? s : os);
    ti[j] = pc ? pi : (c ? v : oi);
    pc = c;
    ps = os;
    pi = oi;
  }
}

// r[j] for a run-time j in [0, 8).
__device__ __forceinline__ uint32_t select8(const uint32_t* r, int j) {
  const uint32_t a0 = (j & 1) ? r[1] : r[0], a1 = (j & 1) ? r[3] : r[2];
  const uint32_t a2 = (j & 1) ? r[5] : r[4], a3 = (j & 1) ? r[7] : r[6];
  const uint32_t b0 = (j & 2) ? a1 : a0, b1 = (j & 2) ? a3 : a2;
  return (j & 4) ? b1 : b0;
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
  __shared__ double2 atab[kAngleTableEntries];
  enc::angle_tables(1 << a.L.b_theta, a.atab, atab, threadIdx.x, blockDim.x);
  __syncthreads();
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
    encode_vector_any<D>(a.L, a.signs, a.St, atab, a.inv_sqrt_d, a.status, load, true, rbuf, codes, bits,
                         sc, sc + 1);
    const int64_t g = a.start + v;
    // group g / 32, chunk-major: byte b of vector g at chunk b / 16
    uint8_t* grp = a.codes + (g >> 5) * (32 * P) + (g & 31) * 16;
#pragma unroll
    for (int k = 0; k < PL; ++k) {
      const int b = lane * PL + k;
      grp[(b >> 4) * 512 + (b & 15)] = codes[b];
    }
    if (lane < 8)
      *reinterpret_cast<uint32_t*>(a.signs_out + (g >> 5) * 1024 + (lane >> 2) * 512 + (g & 31) * 16 +
                                   (lane & 3) * 4) = bits[lane];
    if (lane == 0) {
      a.s16_out[g] = sc[0];
      a.rn16_out[g] = sc[1];
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// query prep: 8 query rows per CTA of 256 threads (rows past nq are written
// as zeros).  Each warp rotates one query (q' = R q); then thread i forms
// q''_i = sum_j S_ij q'_j for the 8 queries (each element of S^T read once
// per CTA, four q' values per shared load); then each warp scales and writes
// its row.
// ---------------------------------------------------------------------------
constexpr int kQpRows = 8;

template <int D>
__global__ void __launch_bounds__(256) vec_qprep_kernel(const VecQPrepArgs a) {
  constexpr int E = D / 32;
  extern __shared__ float qsm[];
  float* sq = qsm;                       // [8][D]   q'
  float* sqq = qsm + kQpRows * D;        // [8][256] q''
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q0 = blockIdx.x * kQpRows;
  for (int rq = warp; rq < kQpRows; rq += 8) {
    const int q = q0 + rq;
    const bool live = q < a.nq;
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int j = lane * E + i;
      x[i] = (live && j < a.dim) ? a.q[(size_t)q * a.dim + j] * (float)a.signs[j] : 0.f;
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
#pragma unroll
    for (int i = 0; i < E; ++i) sq[rq * D + lane * E + i] = x[i] * inv;
  }
  __syncthreads();
  {
    const int i = threadIdx.x;           // output index of q''
    float acc[kQpRows];
#pragma unroll
    for (int r = 0; r < kQpRows; ++r) acc[r] = 0.f;
    if (i < a.m) {
      for (int j = 0; j < D; j += 4) {
        float sv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) sv[e] = __ldg(a.St + (size_t)(j + e) * a.m + i);
#pragma unroll
        for (int r = 0; r < kQpRows; ++r) {
          const float4 x = *reinterpret_cast<const float4*>(sq + r * D + j);
          acc[r] = fmaf(sv[0], x.x, acc[r]);
          acc[r] = fmaf(sv[1], x.y, acc[r]);
          acc[r] = fmaf(sv[2], x.z, acc[r]);
          acc[r] = fmaf(sv[3], x.w, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kQpRows; ++r) sqq[r * 256 + i] = acc[r];
  }
  __syncthreads();
  const int ka = D + 16 * a.kq;
  for (int rq = warp; rq < kQpRows; rq += 8) {
    const int q = q0 + rq;
    const float* xq = sq + rq * D;
    const float* xqq = sqq + rq * 256;
    float amax = 0.f;
    for (int k = lane; k < D; k += 32) amax = fmaxf(amax, fabsf(xq[k]));
    for (int k = lane; k < a.m; k += 32) amax = fmaxf(amax, fabsf(xqq[k]));
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float al = amax > 0.f ? exp2f(-floorf(log2f(amax))) : 1.f;
    // row q of the operand: D polar columns, then kq k-steps of QJL columns
    __half* row = a.A + (size_t)q * ka;
    for (int k = lane; k < D; k += 32) row[k] = __float2half_rn(xq[k] * al);
    for (int c = lane; c < a.kq * 16; c += 32) {
      const int t = c >> 4, kc = (c >> 3) & 1, u = (c >> 1) & 3, e = c & 1;
      const int h = (t == a.kq - 1 && a.half_last) ? 1 : (t & 1);
      const int up = 8 * h + 4 * kc + u;
      const int bit = 32 * (t >> 1) + (e ? 31 - up : 15 - up);
      row[D + c] = __float2half_rn(bit < a.m ? xqq[bit] * al : 0.f);
    }
    if (q < a.nq && lane == 0) a.qscale[q] = 1.f / al;
  }
}

// ---------------------------------------------------------------------------
// search
// ---------------------------------------------------------------------------
// Rounds of kN database vectors; each round's k-steps (D/16 polar, then kq
// QJL) pass through a ring of NB B stages of KSTG k-steps:
//   producers  --full[slot]-->  MMA thread  --empty[slot] (commit)-->  producers
//   MMA thread --acc_full[b] (commit)--> epilogue group b --acc_empty[b]--> MMA thread
// Round r accumulates in tensor-memory columns [kN (r % 2), kN (r % 2 + 1));
// epilogue group g (warps 4g .. 4g + 3) reads the round's columns
// [kN/2 g, kN/2 (g + 1)), so each query keeps two best lists, one per
// column half.  Every wait is bounded;
// a timeout raises the CTA's abort flag, which ends every role's loop, and
// the kernel still waits for its issued MMAs and frees its tensor memory
// before it returns.
template <int D>
__global__ void __launch_bounds__(kSearchThreads, 1) search_umma_kernel(const SearchArgs a) {
  using U = SearchSmem;
  constexpr int KP = D / 16;      // polar k-steps
  constexpr int PC = D / 64;      // polar chunks (16 code bytes) per producer thread
  constexpr int KSTG = D >= 128 ? 8 : 4;   // k-steps per stage
  constexpr int NB = kRingKSteps / KSTG;   // stages in the ring
  constexpr int CPS = KSTG / 4;            // chunks (or sign words) per producer thread per stage
  constexpr int STAGE_BYTES = KSTG * kKStepB;
  static_assert(KP % KSTG == 0 && NB <= kMaxStages, "polar k-steps fill whole stages");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = KP + a.kq;
  const int nst = (ks + KSTG - 1) / KSTG;   // stages per round
  const uint32_t sbase = smem_addr(smem);
  const uint32_t b_s = sbase + U::B;
  const uint32_t bar_full = sbase + U::BAR, bar_empty = bar_full + 8 * kMaxStages;
  const uint32_t bar_accf = bar_empty + 8 * kMaxStages, bar_acce = bar_accf + 16, bar_done = bar_acce + 16;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + U::ABORT);

  // this CTA's run: rounds [r0, r1) of the database
  const int64_t rounds = (a.n + kN - 1) / kN;
  const int64_t r0 = rounds * blockIdx.y / gridDim.y, r1 = rounds * (blockIdx.y + 1) / gridDim.y;
  const int nr = (int)(r1 - r0);
  const int64_t v_lo = r0 * kN;
  const int64_t v_hi = r1 * kN < a.n ? r1 * kN : a.n;

  // LUT of c_r * (cos, sin)(2 pi c_th / 2^b_th), one copy per lane
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + U::LUT);
  for (int e = tid; e < 256 * 32; e += blockDim.x) {
    const int w = e >> 5;
    const int cr = w >> a.b_theta, ct = w & ((1 << a.b_theta) - 1);
    float sn, cs;
    sincospif(2.0f * (float)ct / (float)(1 << a.b_theta), &sn, &cs);
    const __half2 h = __floats2half2_rn((float)cr * cs, (float)cr * sn);
    lut[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  if (tid == 0) {
    for (int i = 0; i < NB; ++i) {
      mbar_init(bar_full + 8 * i, kProdWarps);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_accf + 8 * i, 1);
      mbar_init(bar_acce + 8 * i, kEpiWarps);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(sbase + U::TMEM_SLOT, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + U::TMEM_SLOT);
  // A: warps 0-3 copy their 32 query rows into tensor memory, one k-step
  // (8 columns) per store
  if (warp < 4) {
    const uint4* src = reinterpret_cast<const uint4*>(a.A + ((size_t)blockIdx.x * kM + 32 * warp + lane) * (16 * ks));
    const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + kTmemA;
    for (int s = 0; s < ks; ++s) {
      const uint4 x0 = src[2 * s], x1 = src[2 * s + 1];
      const uint32_t r[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      tmem_st8(ta + 8 * s, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp < kEpiWarps) {
    // ---------------- epilogue: thread = query row 32 (warp % 4) + lane ----
    // warp group g = warp / 4 reads columns [64 g, 64 g + 64) of every round
    const int quarter = warp & 3, grp = warp >> 2;
    const int qr = 32 * quarter + lane;
    float ts[kListK];
    int ti[kListK];
#pragma unroll
    for (int j = 0; j < kListK; ++j) {
      ts[j] = kNegInf;
      ti[j] = 0x7fffffff;
    }
    float thr = kNegInf;
    int cnt = 0;
    const uint32_t qbase = sbase + U::QUEUE + (uint32_t)(32 * warp + lane) * 8;   // entry i at + i * 2048
    constexpr uint32_t kQStride = kEpiWarps * 32 * 8;
    auto flush = [&]() {
      const int mx = __reduce_max_sync(kFull, cnt);
      for (int i = 0; i < mx; ++i) {
        if (i < cnt) {
          const float2 c = lds64f(qbase + i * kQStride);
          list_insert<kListK>(ts, ti, c.x, __float_as_int(c.y));
        }
      }
      cnt = 0;
      thr = ts[kListK - 1];
    };
    const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(grp * (kN / 2));
    for (int r = 0; r < nr; ++r) {
      const int ab = r & 1;
      if (!warp_wait(bar_accf + 8 * ab, (uint32_t)((r >> 1) & 1), a.wait_limit_ns, abort_flag, a.status))
        break;
      tc_fence_after();
      const int64_t vr = v_lo + (int64_t)r * kN;
      const int valid = (int)(v_hi - vr < kN ? v_hi - vr : kN);
#pragma unroll 1
      for (int c = 0; c < kN / 64; ++c) {
        uint32_t sv[32];
        tmem_ld32(taddr + (uint32_t)(ab * kN + 32 * c), sv);
        const float* f = reinterpret_cast<const float*>(sv);
        const int col0 = grp * (kN / 2) + 32 * c;
        // sub-chunks of 8 columns holding a score above the lane's threshold
        uint32_t hit = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float mx = fmaxf(max3f(f[8 * t], f[8 * t + 1], f[8 * t + 2]),
                                 max3f(max3f(f[8 * t + 3], f[8 * t + 4], f[8 * t + 5]), f[8 * t + 6], f[8 * t + 7]));
          hit |= (mx > thr && col0 + 8 * t < valid) ? (1u << t) : 0u;
        }
        const uint32_t any = __reduce_or_sync(kFull, hit);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (!(any & (1u << t))) continue;
          const int col = col0 + 8 * t;
          uint32_t m = 0;
#pragma unroll
          for (int u = 0; u < 8; ++u) m |= (f[8 * t + u] > thr ? 1u : 0u) << u;
          const int nv = valid - col;
          if (nv < 8) m &= (1u << nv) - 1u;
          while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            sts64f(qbase + cnt * kQStride, __uint_as_float(select8(sv + 8 * t, j)),
                   __int_as_float((int)(vr + col + j)));
            ++cnt;
          }
          if (__any_sync(kFull, cnt > kQ - 8)) flush();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acce + 8 * ab);
    }
    flush();
    const int q = blockIdx.x * kM + qr;
    if (q < a.nq) {
      const size_t base = (((size_t)q * gridDim.y + blockIdx.y) * 2 + grp) * kListK;
#pragma unroll
      for (int j = 0; j < kListK; ++j) {
        a.part_s[base + j] = ts[j];
        a.part_i[base + j] = ti[j];
      }
    }
  } else if (warp < kMmaWarp) {
    // ---------------- producers --------------------------------------------
    // thread: vector n of each round; half h takes the polar chunks c with
    // c % 2 == h (k-steps 2c, 2c + 1) and the sign words w with w % 2 == h
    // (QJL k-steps 2w, 2w + 1): k-steps 4i + 2h, 4i + 2h + 1 (i < KSTG / 4)
    // of every stage.
    const int pw = warp - kEpiWarps;
    const int h = pw >> 2;
    const int n = 32 * (pw & 3) + lane;
    const uint32_t row_off = (uint32_t)((n >> 3) * 256 + (n & 7) * 16);   // core-matrix row of vector n
    const uint32_t* lutp = lut + lane;
    uint32_t cw[4 * PC], sg[4];
    uint32_t ncw[4 * PC], nsg[4];
    uint32_t raw_s = 0, raw_r = 0, nraw_s = 0, nraw_r = 0;   // s16, rn16 bits
    auto load = [&](int r, uint32_t (&w)[4 * PC], uint32_t (&g)[4], uint32_t& xs, uint32_t& xr) {
      const int64_t v = v_lo + (int64_t)r * kN + n;
      if (r < nr && v < v_hi) {
        const int64_t grp = v >> 5;                // lane == v % 32
        const uint8_t* cp = a.codes + grp * (32 * (D / 2)) + 16 * lane;
#pragma unroll
        for (int i = 0; i < PC; ++i)
          ldg_stream4(cp + 512 * (2 * i + h), w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        // sign words h, 2 + h (chunk 0) and 4 + h, 6 + h (chunk 1)
        const uint8_t* sp = a.signs + grp * 1024 + 16 * lane + 4 * h;
        ldg_stream1(sp, g[0]);
        ldg_stream1(sp + 8, g[1]);
        ldg_stream1(sp + 512, g[2]);
        ldg_stream1(sp + 520, g[3]);
        ldg_stream_u16(a.s16 + v, xs);
        ldg_stream_u16(a.rn16 + v, xr);
      } else {
#pragma unroll
        for (int c = 0; c < 4 * PC; ++c) w[c] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) g[c] = 0u;
        xs = 0u;                                   // columns past the run score 0 (masked later)
        xr = 0u;
      }
    };
    load(0, cw, sg, raw_s, raw_r);
    uint32_t slot = 0, phase = 0;
    auto acquire = [&]() {
      return warp_wait(bar_empty + 8 * slot, phase ^ 1u, a.wait_limit_ns, abort_flag, a.status);
    };
    auto release = [&]() {
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_full + 8 * slot);
      if (++slot == NB) {
        slot = 0;
        phase ^= 1u;
      }
    };
    auto kstep_ptr = [&](int j) {          // this thread's row of k-step j of the current stage
      return reinterpret_cast<uint4*>(smem + U::B + slot * STAGE_BYTES + j * kKStepB + row_off);
    };
    for (int r = 0; r < nr; ++r) {
      load(r + 1, ncw, nsg, nraw_s, nraw_r);
      // the scales loaded a round ago: s16/(2^b_r-1) for the polar values,
      // -rn16 sqrt(pi/2)/m for the QJL ones (a set sign bit makes it +)
      uint32_t sa, sb;
      {
        const float s16 = __half2float(__ushort_as_half((unsigned short)raw_s));
        const float rn = __half2float(__ushort_as_half((unsigned short)raw_r));
        const uint32_t au = __half_as_ushort(__float2half_rn(s16 * a.inv_levels));
        const uint32_t bu = __half_as_ushort(__float2half_rn(rn * a.qjl_const));
        sa = au | (au << 16);
        sb = (bu | (bu << 16)) | 0x80008000u;
      }
      // polar stages: chunk 2i + h (i = CPS st + i2) -> k-steps 4 i2 + 2h + e
#pragma unroll
      for (int st = 0; st < KP / KSTG; ++st) {
        if (!acquire()) goto producers_done;
#pragma unroll
        for (int i2 = 0; i2 < CPS; ++i2) {
          const int i = CPS * st + i2;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            uint4* dst = kstep_ptr(4 * i2 + 2 * h + e);
#pragma unroll
            for (int kc = 0; kc < 2; ++kc) {
              const uint32_t w = cw[4 * i + 2 * e + kc];
              uint32_t q4[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) q4[u] = hmul2_u32(lutp[__byte_perm(w, 0u, 0x4440u + u) << 5], sa);
              dst[kc * 8] = make_uint4(q4[0], q4[1], q4[2], q4[3]);
            }
          }
        }
        release();
      }
      // QJL stages: word 2 (CPS qs + i2) + h -> k-steps t = KSTG qs + 4 i2 + 2h + e
#pragma unroll
      for (int qs = 0; qs < 16 / KSTG; ++qs) {
        if (KSTG * qs < a.kq) {
          if (!acquire()) goto producers_done;
#pragma unroll
          for (int i2 = 0; i2 < CPS; ++i2) {
            const uint32_t x = sg[CPS * qs + i2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int t = KSTG * qs + 4 * i2 + 2 * h + e;
              if (t < a.kq) {
                const int hw = (t == a.kq - 1 && a.half_last) ? 1 : e;
                uint4* dst = kstep_ptr(4 * i2 + 2 * h + e);
#pragma unroll
                for (int kc = 0; kc < 2; ++kc) {
                  const int u0 = 8 * hw + 4 * kc;
                  dst[kc * 8] = make_uint4(((x << u0) & 0x80008000u) ^ sb, ((x << (u0 + 1)) & 0x80008000u) ^ sb,
                                           ((x << (u0 + 2)) & 0x80008000u) ^ sb, ((x << (u0 + 3)) & 0x80008000u) ^ sb);
                }
              }
            }
          }
          release();
        }
      }
#pragma unroll
      for (int c = 0; c < 4 * PC; ++c) cw[c] = ncw[c];
#pragma unroll
      for (int c = 0; c < 4; ++c) sg[c] = nsg[c];
      raw_s = nraw_s;
      raw_r = nraw_r;
    }
  producers_done:;
  } else {
    // ---------------- MMA issue (warp kMmaWarp; one elected lane issues) ----
    uint32_t elected;
    asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n" : "=r"(elected));
    uint32_t slot = 0, phase = 0;
    for (int r = 0; r < nr; ++r) {
      const int ab = r & 1;
      if (!warp_wait(bar_acce + 8 * ab, (uint32_t)(((r >> 1) & 1) ^ 1), a.wait_limit_ns, abort_flag, a.status))
        break;
      tc_fence_after();
      const uint32_t d_t = tmem + (uint32_t)(ab * kN);
      bool ok = true;
      for (int st = 0; st < nst; ++st) {
        if (!warp_wait(bar_full + 8 * slot, phase, a.wait_limit_ns, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int s0 = st * KSTG;
        const int n_in = ks - s0 < KSTG ? ks - s0 : KSTG;
        if (elected) {
          for (int j = 0; j < n_in; ++j)
            umma_f16_ts(d_t, tmem + kTmemA + 8 * (s0 + j), umma_desc(b_s + slot * STAGE_BYTES + j * kKStepB),
                        kIdesc, (s0 + j) > 0 ? 1u : 0u);
          umma_commit(bar_empty + 8 * slot);
        }
        __syncwarp();
        if (++slot == NB) {
          slot = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (elected) umma_commit(bar_accf + 8 * ab);
      __syncwarp();
    }
    // every issued MMA has finished before tensor memory is freed
    if (elected) {
      umma_commit(bar_done);
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bar_done, 0u))
        if (global_ns() - t0 > a.wait_limit_ns) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One warp per query: the k best of its candidate lists (each sorted by
// (score desc, index asc), padded with (-inf, INT_MAX)).  Lane l holds the
// heads of lists l and l + 32; each of the k rounds takes the warp's best
// head and advances that list.
template <int K>
__global__ void __launch_bounds__(256) topk_merge_kernel(const MergeArgs a) {
  const int lane = threadIdx.x & 31;
  const int q = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (q >= a.nq) return;
  const int lists = a.nsplit;
  const size_t base = (size_t)q * lists * K;
  int pos[2] = {0, 0};
  float hs[2];
  int hi[2];
  auto head = [&](int h) {
    const int l = lane + 32 * h;
    if (l < lists && pos[h] < K) {
      hs[h] = a.part_s[base + (size_t)l * K + pos[h]];
      hi[h] = a.part_i[base + (size_t)l * K + pos[h]];
    } else {
      hs[h] = kNegInf;
      hi[h] = 0x7fffffff;
    }
  };
  head(0);
  head(1);
  const float sc = a.qscale[q];
  for (int j = 0; j < a.k; ++j) {
    const int mine = better(hs[1], hi[1], hs[0], hi[0]) ? 1 : 0;
    float bs = hs[mine];
    int bi = hi[mine];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float os = __shfl_xor_sync(kFull, bs, o);
      const int oi = __shfl_xor_sync(kFull, bi, o);
      if (better(os, oi, bs, bi)) {
        bs = os;
        bi = oi;
      }
    }
    // database indices are unique across the lists: one lane owns the winner
    if (bs == hs[mine] && bi == hi[mine] && bi != 0x7fffffff) {
      ++pos[mine];
      head(mine);
    }
    if (lane == 0) {
      a.scores[(size_t)q * a.k + j] = bs * sc;
      a.idx[(size_t)q * a.k + j] = bi;
    }
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
  const size_t smem = SearchSmem::BYTES;
  if (cudaFuncSetAttribute(search_umma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  dim3 grid((a.nq + kM - 1) / kM, a.nsplit);
  search_umma_kernel<D><<<grid, kSearchThreads, smem, s>>>(a);
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

template <int D>
cudaError_t launch_vec_qprep_d(const VecQPrepArgs& a, cudaStream_t s) {
  const int grid = (a.nq + kM - 1) / kM * (kM / kQpRows);     // whole 128-row tiles
  const size_t smem = sizeof(float) * kQpRows * (D + 256);
  if (cudaFuncSetAttribute(vec_qprep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  vec_qprep_kernel<D><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_vec_qprep(const VecQPrepArgs& a, cudaStream_t s) {
  switch (a.d) {
    case 64: return launch_vec_qprep_d<64>(a, s);
    case 128: return launch_vec_qprep_d<128>(a, s);
    case 256: return launch_vec_qprep_d<256>(a, s);
  }
  return cudaErrorInvalidValue;
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
  topk_merge_kernel<kListK><<<(a.nq + 7) / 8, 256, 0, s>>>(a);
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
  const size_t groups = (size_t)((n + 31) / 32);            // whole groups of 32 vectors
  l.codes = off; off += vround(groups * 32 * (d / 2));
  l.signs = off; off += vround(groups * 32 * 32);
  l.s16 = off;   off += vround((size_t)n * 2);
  l.rn16 = off;  off += vround((size_t)n * 2);
  l.total = off;
  return l;
}

struct VecWsLayout {
  size_t status, signs, St, atab, A, qscale, part_s, part_i, total;
};

VecWsLayout vec_ws_layout(int d, int m, int max_q) {
  VecWsLayout w{};
  size_t off = 0;
  w.status = off; off += kVAlign;
  w.signs = off;  off += vround(sizeof(double) * d);
  w.St = off;     off += vround(sizeof(float) * (size_t)d * m);
  w.atab = off;   off += vround(sizeof(double) * 2 * kAngleTableEntries);
  w.A = off;      off += vround((size_t)((max_q + kM - 1) / kM) * kM * (d + 16 * search_qjl_steps(m)) * 2);
  w.qscale = off; off += vround(sizeof(float) * max_q);
  w.part_s = off; off += vround(sizeof(float) * (size_t)max_q * kMaxSplits * 2 * kListK);
  w.part_i = off; off += vround(sizeof(int) * (size_t)max_q * kMaxSplits * 2 * kListK);
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
  std::vector<double> atab(2 * kAngleTableEntries, 0.0);
  angle_table_host(1 << cfg->b_theta, atab.data());
  if (e == cudaSuccess) e = cudaMemcpyAsync(v->ws + v->W.atab, atab.data(), sizeof(double) * atab.size(), cudaMemcpyHostToDevice, stream);
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
  if (!v || !codes || start < 0 || count < 0 || start + count > v->n || ((uintptr_t)codes % kVAlign))
    return TQ_ERR_INVALID_ARG;
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
  a.atab = (const double2*)(v->ws + v->W.atab);
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
  if (!v || !codes || !q || !scores || !idx || nq < 1 || nq > v->max_q || k < 1 || k > kListK ||
      ((uintptr_t)codes % kVAlign))
    return TQ_ERR_INVALID_ARG;
  VecQPrepArgs qa{};
  qa.q = q;
  qa.nq = nq;
  qa.dim = v->cfg.dim;
  qa.d = v->d;
  qa.m = v->cfg.qjl_bits;
  qa.signs = (const double*)(v->ws + v->W.signs);
  qa.St = (const float*)(v->ws + v->W.St);
  qa.kq = search_qjl_steps(v->cfg.qjl_bits);
  qa.half_last = v->cfg.qjl_bits % 32 == 8 ? 1 : 0;
  qa.A = (__half*)(v->ws + v->W.A);
  qa.qscale = (float*)(v->ws + v->W.qscale);
  if (launch_vec_qprep(qa, stream) != cudaSuccess) return TQ_ERR_CUDA;
  // one wave of one CTA per SM: query tiles x database splits
  const int qtiles = (nq + kM - 1) / kM;
  int nsplit = std::max(1, v->num_sms / qtiles);
  nsplit = std::min(nsplit, kMaxSplits);
  nsplit = (int)std::min<int64_t>(nsplit, (v->n + kN - 1) / kN);
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
  sa.kq = qa.kq;
  sa.half_last = qa.half_last;
  sa.status = (int*)(v->ws + v->W.status);
  sa.wait_limit_ns = kDefaultWaitLimitNs;
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
  ma.nsplit = 2 * nsplit;            // two lists (column halves) per split
  ma.k = k;
  ma.scores = scores;
  ma.idx = idx;
  return launch_topk_merge(ma, stream) == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_vec_get_status(tq_vec_index* v, cudaStream_t stream) {
  if (!v) return TQ_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  int word = 0;
  int* st = (int*)(v->ws + v->W.status);
  if (cudaMemcpy(&word, st, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ERR_CUDA;
  if (word != 0 && cudaMemset(st, 0, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  if (word & kStatusTimeout) return TQ_ERR_TIMEOUT;
  if (word & kStatusRange) return TQ_ERR_RANGE;
  return TQ_OK;
}

tq_status tq_export_vectors(tq_vec_index* v, const void* codes, int64_t start, int64_t count,
                            uint8_t* codes_out, uint8_t* bits_out, uint16_t* s16_out,
                            uint16_t* rn16_out, cudaStream_t stream) {
  if (!v || !codes || start < 0 || count < 0 || start + count > v->n) return TQ_ERR_INVALID_ARG;
  if (count == 0) return TQ_OK;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TQ_ERR_CUDA;
  const uint8_t* base = (const uint8_t*)codes;
  const int P = v->d / 2, mb = v->cfg.qjl_bits / 8;
  // the groups of 32 vectors that hold [start, start + count)
  const int64_t g0 = start / 32, g1 = (start + count + 31) / 32;
  cudaError_t e = cudaSuccess;
  if (codes_out) {
    // bw = 8: the canonical LSB-first stream is one byte per pair
    std::vector<uint8_t> tmp((size_t)(g1 - g0) * 32 * P);
    e = cudaMemcpy(tmp.data(), base + v->C.codes + g0 * 32 * P, tmp.size(), cudaMemcpyDeviceToHost);
    for (int64_t i = 0; e == cudaSuccess && i < count; ++i) {
      const int64_t g = start + i, off = (g / 32 - g0) * 32 * P + (g % 32) * 16;
      for (int b = 0; b < P; ++b) codes_out[i * P + b] = tmp[off + (b / 16) * 512 + b % 16];
    }
  }
  if (e == cudaSuccess && bits_out) {
    std::vector<uint8_t> tmp((size_t)(g1 - g0) * 1024);
    e = cudaMemcpy(tmp.data(), base + v->C.signs + g0 * 1024, tmp.size(), cudaMemcpyDeviceToHost);
    for (int64_t i = 0; e == cudaSuccess && i < count; ++i) {
      const int64_t g = start + i, off = (g / 32 - g0) * 1024 + (g % 32) * 16;
      for (int b = 0; b < mb; ++b) bits_out[i * mb + b] = tmp[off + (b / 16) * 512 + b % 16];
    }
  }
  if (e == cudaSuccess && s16_out) e = cudaMemcpy(s16_out, base + v->C.s16 + start * 2, (size_t)count * 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && rn16_out) e = cudaMemcpy(rn16_out, base + v->C.rn16 + start * 2, (size_t)count * 2, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // extern "C"
