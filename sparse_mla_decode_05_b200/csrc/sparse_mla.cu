// sparse_mla.cu -- sm_100a kernels and C ABI of the sparse-MLA decode library.
//
// Source pages (by title):
//   [Design] "The MMA Sparse-MLA Decode Kernel: A Deep Dive into AI Inference
//            Optimization on Blackwell GPUs"
//   [Truth]  "The Moment of Truth: Analyzing a Custom MMA Kernel's Performance
//            on Blackwell GPUs"
//   [Pivot]  "The Pivot Point: When a 6.3x Kernel Speedup Reveals the Next
//            Bottleneck"
//   [Diag]   "The Moment of Diagnosis: How One GPU Kernel Laid Bare the Ceiling
//            of Blackwell Inference"
//
// What the pages prescribe, and how this file realises it on B200:
//  * Gather each top-k KV tile ONCE and reuse it for all 64 heads, instead of
//    one program per head re-reading the same rows 64 times ([Diag] "The
//    Subject Message"; [Design] "Design Decisions" 1).  Here one CTA owns
//    (sequence, top-k chunk); 64-token tiles are gathered into shared memory
//    with 16-byte cp.async (fp8 rows: register loads + exact fp8->bf16
//    conversion) and consumed by the tensor cores for every head.
//  * Scores and PV as tensor-core contractions across the head group with
//    fp32 accumulation ([Design] "Design Decisions" 5-6).  Here: tcgen05.mma
//    with accumulators in tensor memory (TMEM):
//        S  = Q . K^T     M = 64 heads, N = 64 tokens, K = 576   (TMEM, fp32)
//        O^T += V^T . P^T M = 128 dims (x4 chunks), N = 64 heads, K = 64 tokens
//    The whole 64x576 query lives in shared memory next to two tile buffers:
//    B200's 227 KB per CTA lets BLOCK_H = 64 (all heads) fit, which the
//    pages' ~99 KB sm_120 budget forbade ([Design] "Memory Budgeting").
//  * Online softmax in fp32; masked entries (index -1) take no part
//    ([Design] "Edge Case Handling").  Rows of masked entries are zero-filled
//    in shared memory and their probabilities are exactly 0.
//  * Split-K over the top-k list with a log-sum-exp combine, so that small
//    batches still spread over all SMs; the split count is a pure function of
//    (batch, top-k, SM count) so that the grid is fixed per batch bucket for
//    CUDA-graph capture ([Truth] "The Split-K Solution: Reasoning About the
//    Fix"; [Pivot] "The Reasoning: Weighing Two Paths").
//
// Warp roles in the split kernel (one CTA per SM; ~227 KB shared memory):
//   warps 0-3  softmax + epilogue (128 threads; warp w owns TMEM lanes 32w..)
//   warp  4    TMEM allocator; lane 0 issues every tcgen05.mma
//   warps 5..  producers: resolve indices (flat or paged), gather rows
// Every wait on a pipeline barrier is bounded (about 2 s): on expiry the CTA
// records an error bit in a device word, drains its own copies and MMAs,
// frees TMEM and exits.

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <math.h>

#include "sparse_mla.h"

namespace smla {

// ---------------------------------------------------------------- constants
constexpr int kH = 64;            // heads
constexpr int kDqk = 576;         // query / key width
constexpr int kDv = 512;          // value width (first 512 dims of a row)
constexpr int kTile = 64;         // tokens per tile
constexpr int kAtoms = kDqk / 64; // 64-dim column blocks (128 B of bf16)
constexpr int kAtomBytes = 64 * 128;                // 64 rows x 128 B
constexpr int kTileBytes = kAtoms * kAtomBytes;     // 73,728
constexpr int kRowBytesBf16 = kDqk * 2;             // 1152
constexpr int kRowBytesFp8 = kDqk;                  // 576

// shared memory map (offsets from a 1024-aligned base)
constexpr int kSmemQ = 0;                           // Q   [9 atoms][64 heads][128 B]
constexpr int kSmemKV = kSmemQ + kTileBytes;        // KV  [2 stages][9 atoms][64 tok][128 B]
constexpr int kSmemP = kSmemKV + 2 * kTileBytes;    // P   [64 heads][64 tok] bf16 (K-major)
constexpr int kSmemAux = kSmemP + 64 * 128;
constexpr int kNumBars = 12;
constexpr int kAuxBars = kSmemAux;                  // 12 mbarriers
constexpr int kAuxTmem = kAuxBars + 8 * kNumBars;   // TMEM base address (4 B)
constexpr int kAuxRow = kAuxTmem + 16;              // int  [2][64] physical row or -1
constexpr int kAuxRsc = kAuxRow + 2 * 64 * 4;       // f32  [2][64] fp8 row scales
constexpr int kAuxAlpha = kAuxRsc + 2 * 64 * 4;     // f32  [64] rescale factors
constexpr int kAuxInvl = kAuxAlpha + 64 * 4;        // f32  [64] 1/l
constexpr int kAuxLse = kAuxInvl + 64 * 4;          // f32  [64] lse
constexpr int kAuxEnd = kAuxLse + 64 * 4;
constexpr int kSmemBytes = kAuxEnd + 1024;          // + alignment slack
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-CTA shared memory of sm_100");

// barrier indices
constexpr int BAR_Q = 0, BAR_KVF = 1, BAR_KVE = 3, BAR_SF = 5, BAR_SE = 7, BAR_PF = 9,
              BAR_PVD = 10, BAR_FIN = 11;

// TMEM columns (512 allocated): O^T chunks at 0..255, S buffers at 256 and 320
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;

// Lazy rescaling: keep the running max until a new max exceeds it by more
// than 2^8 (probabilities stay <= 256; results are unchanged).
constexpr float kRescaleThresh = 8.0f;

// Instruction descriptors (kind::f16): D f32 (bits 4-5 = 1), A bf16 (7-9 = 1),
// B bf16 (10-12 = 1), A major bit 15, B major bit 16, N>>3 at 17, M>>4 at 24.
constexpr uint32_t make_idesc(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescS = make_idesc(64, 64, false, false);    // S  = Q K^T
constexpr uint32_t kIdescPV = make_idesc(128, 64, true, false);   // O^T = V^T P^T

constexpr unsigned long long kWaitLimitNs = 2000000000ull;

template <bool kFp8>
struct Cfg {
  static constexpr int kProdWarps = kFp8 ? 8 : 4;
  static constexpr int kProdThreads = kProdWarps * 32;
  static constexpr int kThreads = (4 + 1 + kProdWarps) * 32;
};

struct SplitParams {
  const uint8_t* q;            // [B, 64, 576] bf16
  const uint8_t* kv;           // rows of 1152 B (bf16) or 576 B (fp8 codes)
  const float* kv_row_scale;   // [N] (fp8)
  const int32_t* page_table;   // [B, pages_per_seq] (paged)
  const int32_t* indices;      // [B, topk]
  __nv_bfloat16* out;          // [B, 64, 512]
  float* lse;                  // [B, 64]
  float* part_o;               // [B, nsplit, 64, 512]
  float* part_lse;             // [B, nsplit, 64]
  int batch, topk, nsplit, ntiles_total;
  int page_size, pages_per_seq;
  float scale_log2;            // scale * log2(e)
};

__device__ unsigned int g_error_word = 0;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking probe (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false (and an error bit) if the phase did not complete in time.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_error_word, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// true in every participating thread iff `pred` holds in any of them
__device__ __forceinline__ bool group_any(bool pred, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_global_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// two fp32 -> packed bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// two fp8 e4m3fn codes (low byte first) -> packed bf16x2, exact
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
  const float lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  const float hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
  return pack_bf16x2(lo, hi);
}

// ---- tcgen05 (5th-generation tensor cores, tensor memory)
__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem desc] . B[smem desc]
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16 lanes x 32 columns, twice: threads 0-15 read columns [c, c+32) of lanes
// base+0..15, threads 16-31 read columns [c+32, c+64) of the same lanes.
__device__ __forceinline__ void tmem_ld_16x32bx2_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 32 bits x 32 columns: thread t reads lane base+t, columns [c, c+32)
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start
// address, leading/stride byte offsets >> 4, version 1 at bit 46, layout
// type 2 = SWIZZLE_128B at bits 61-63).
//  K-major operand  (rows of 128 B, 8-row groups 1024 B apart): lbo unused.
//  MN-major operand (64-element MN blocks `lbo` apart, 8-row K groups `sbo`).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// byte offset of 16-byte chunk `j` (0..7) of row `r` in a 128B-swizzled block
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
  return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

// ============================================================ split kernel
template <bool kFp8>
__global__ void __launch_bounds__(Cfg<kFp8>::kThreads, 1)
    smla_split_kernel(const __grid_constant__ SplitParams p) {
  constexpr int kProd = Cfg<kFp8>::kProdThreads;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kAuxBars;
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y;
  const int t_begin = (int)((long long)split * p.ntiles_total / p.nsplit);
  const int t_end = (int)((long long)(split + 1) * p.ntiles_total / p.nsplit);
  const int ntiles = t_end - t_begin;
  const int tok_begin = t_begin * kTile;
  const int tok_end = min(t_end * kTile, p.topk);

  int* s_row = reinterpret_cast<int*>(smem + kAuxRow);
  float* s_rsc = reinterpret_cast<float*>(smem + kAuxRsc);
  float* s_alpha = reinterpret_cast<float*>(smem + kAuxAlpha);
  float* s_invl = reinterpret_cast<float*>(smem + kAuxInvl);
  float* s_lse = reinterpret_cast<float*>(smem + kAuxLse);

  if (threadIdx.x == 0) {
    mbar_init(BAR(BAR_Q), kProd);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(BAR_KVF + s), kFp8 ? kProd : 2 * kProd);
      mbar_init(BAR(BAR_KVE + s), 1);
      mbar_init(BAR(BAR_SF + s), 1);
      mbar_init(BAR(BAR_SE + s), 128);
    }
    mbar_init(BAR(BAR_PF), 128);
    mbar_init(BAR(BAR_PVD), 1);
    mbar_init(BAR(BAR_FIN), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 4) {
    tmem_alloc(sbase + kAuxTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kAuxTmem);

  if (warp >= 5) {
    // ------------------------------------------------------------ producers
    const int ptid = threadIdx.x - 160;
    {  // the 64 x 576 query, once, into the 128B-swizzled K-major layout
      const uint8_t* qsrc = p.q + (size_t)b * kH * kRowBytesBf16;
      for (int c = ptid; c < kH * 72; c += kProd) {
        const int h = c / 72, ch = c - h * 72;
        const uint32_t dst = sbase + kSmemQ + (ch >> 3) * kAtomBytes + sw128_off(h, ch & 7);
        cp_async_16(dst, qsrc + (size_t)h * kRowBytesBf16 + ch * 16, 16);
      }
      cp_async_mbar_arrive_noinc(BAR(BAR_Q));
    }
    for (int t = 0; t < ntiles; ++t) {
      const int slot = t & 1;
      bool fail = false;
      if (t >= 2) fail = !mbar_wait(BAR(BAR_KVE + slot), ((t >> 1) - 1) & 1);
      if (group_any(fail, 1, kProd)) break;
      if (ptid < kTile) {  // index -> physical row (or -1)
        const int pos = tok_begin + t * kTile + ptid;
        int row = -1;
        float rs = 0.f;
        if (pos < tok_end) {
          const int idx = p.indices[(size_t)b * p.topk + pos];
          if (idx >= 0) {
            row = p.page_size ? p.page_table[(size_t)b * p.pages_per_seq + idx / p.page_size] * p.page_size +
                                    idx % p.page_size
                              : idx;
            if (kFp8) rs = p.kv_row_scale[row];
          }
        }
        s_row[slot * kTile + ptid] = row;
        if (kFp8) s_rsc[slot * kTile + ptid] = rs;
      }
      named_bar_sync(1, kProd);
      const uint32_t tbase = sbase + kSmemKV + slot * kTileBytes;
      if constexpr (!kFp8) {
        // 64 rows x 72 chunks of 16 B; consecutive lanes take consecutive
        // chunks of a row (coalesced); padding rows are zero-filled.
        for (int c = ptid; c < kTile * 72; c += kProd) {
          const int tok = c / 72, ch = c - tok * 72;
          const int row = s_row[slot * kTile + tok];
          const uint8_t* src = p.kv + (size_t)(row >= 0 ? row : 0) * kRowBytesBf16 + ch * 16;
          cp_async_16(tbase + (ch >> 3) * kAtomBytes + sw128_off(tok, ch & 7), src, row >= 0 ? 16u : 0u);
        }
        cp_async_mbar_arrive_noinc(BAR(BAR_KVF + slot));
        mbar_arrive(BAR(BAR_KVF + slot));
      } else {
        // 64 rows x 36 chunks of 16 fp8 codes; all loads issued first, then
        // converted exactly to bf16 and stored swizzled.
        constexpr int kPer = kTile * 36 / kProd;
        static_assert(kTile * 36 % kProd == 0, "fp8 producer split");
        uint4 v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int c = ptid + u * kProd;
          const int tok = c / 36, ch = c - tok * 36;
          const int row = s_row[slot * kTile + tok];
          v[u] = row >= 0 ? ld_global_nc_v4(p.kv + (size_t)row * kRowBytesFp8 + ch * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int c = ptid + u * kProd;
          const int tok = c / 36, ch = c - tok * 36;
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          uint4 lo, hi;
          lo.x = e4m3x2_to_bf16x2((uint16_t)(w[0] & 0xFFFF));
          lo.y = e4m3x2_to_bf16x2((uint16_t)(w[0] >> 16));
          lo.z = e4m3x2_to_bf16x2((uint16_t)(w[1] & 0xFFFF));
          lo.w = e4m3x2_to_bf16x2((uint16_t)(w[1] >> 16));
          hi.x = e4m3x2_to_bf16x2((uint16_t)(w[2] & 0xFFFF));
          hi.y = e4m3x2_to_bf16x2((uint16_t)(w[2] >> 16));
          hi.z = e4m3x2_to_bf16x2((uint16_t)(w[3] & 0xFFFF));
          hi.w = e4m3x2_to_bf16x2((uint16_t)(w[3] >> 16));
          // dims [16ch, 16ch+16) = bf16 chunks 2ch, 2ch+1 of the row
          const int j0 = (ch & 3) * 2;
          const uint32_t rb = tbase + (ch >> 2) * kAtomBytes;
          st_shared_v4(rb + sw128_off(tok, j0), lo);
          st_shared_v4(rb + sw128_off(tok, j0 + 1), hi);
        }
        fence_proxy_async_smem();
        mbar_arrive(BAR(BAR_KVF + slot));
      }
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(BAR(BAR_Q), 0);
      int ns = 0, npv = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok && npv < ntiles) {
        bool progressed = false;
        if (ns < ntiles && ns <= npv + 1) {
          const int slot = ns & 1;
          if (mbar_test_wait(BAR(BAR_KVF + slot), (ns >> 1) & 1) &&
              (ns < 2 || mbar_test_wait(BAR(BAR_SE + slot), ((ns >> 1) - 1) & 1))) {
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t qa = sbase + kSmemQ;
            const uint32_t ka = sbase + kSmemKV + slot * kTileBytes;
            const uint32_t d = tmem + kColS + 64u * (uint32_t)slot;
#pragma unroll 4
            for (int k = 0; k < kDqk / 16; ++k) {
              const uint32_t off = (k >> 2) * kAtomBytes + (k & 3) * 32;
              mma_bf16(d, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), kIdescS,
                       k > 0 ? 1u : 0u);
            }
            tc_commit(BAR(BAR_SF + slot));
            ++ns;
            progressed = true;
          }
        }
        if (npv < ns && mbar_test_wait(BAR(BAR_PF), npv & 1)) {
          tc_fence_after();
          const int slot = npv & 1;
          const uint32_t va = sbase + kSmemKV + slot * kTileBytes;
          const uint32_t pa = sbase + kSmemP;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_bf16(tmem + kColO + 64u * (uint32_t)c,
                       sw128_desc(va + (2 * c) * kAtomBytes + kk * 2048, kAtomBytes, 1024),
                       sw128_desc(pa + kk * 32, 16, 1024), kIdescPV, (npv > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(BAR(BAR_KVE + slot));
          tc_commit(BAR(BAR_PVD));
          ++npv;
          progressed = true;
        }
        if (progressed) {
          t_last = globaltimer_ns();
        } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
          atomicOr(&g_error_word, 1u);
          ok = false;
        }
      }
      // drain: every MMA this thread issued has completed before teardown
      tc_commit(BAR(BAR_FIN));
      mbar_wait(BAR(BAR_FIN), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int h = 16 * warp + (lane & 15);   // head row of this thread
    const int half = lane >> 4;              // tokens [32*half, 32*half+32)
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    // l_run: sum of the probabilities as fp32 (gives lse); l_pv: the same sum
    // of the bf16-rounded probabilities the PV MMA used (normalises out, so
    // the output weights sum to one exactly).  fp8 rows fold the row scale
    // into P, so there l_pv = l_run.
    float m_run = -INFINITY, l_run = 0.f, l_pv = 0.f;
    bool aborted = false;
    for (int i = 0; i < ntiles; ++i) {
      const int sb = i & 1;
      // S(i) is in TMEM; the load barrier of the tile is complete too (S
      // consumed it), and waiting on it here acquires the producers' row
      // table and row scales for this tile.
      const bool f1 = !mbar_wait(BAR(BAR_SF + sb), (i >> 1) & 1) || !mbar_wait(BAR(BAR_KVF + sb), (i >> 1) & 1);
      if (group_any(f1, 2, 128)) { aborted = true; break; }
      tc_fence_after();
      float s[32];
      tmem_ld_16x32bx2_x32(tmem + lane_base + kColS + 64u * (uint32_t)sb, s);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(BAR_SE + sb));

      const int* rows = s_row + sb * kTile + half * 32;
      const float* rsc = s_rsc + sb * kTile + half * 32;
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float f = kFp8 ? p.scale_log2 * rsc[j] : p.scale_log2;
        const float x = rows[j] >= 0 ? s[j] * f : -INFINITY;
        s[j] = x;
        tmax = fmaxf(tmax, x);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
      const float m_new = fmaxf(m_run, tmax);
      const bool need = m_new > m_run + kRescaleThresh;
      const float m_use = need ? m_new : m_run;
      const float alpha = need ? ex2(m_run - m_use) : 1.f;
      uint32_t pk[16];
      float lsum = 0.f, lsum_pv = 0.f;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float p0 = s[j] == -INFINITY ? 0.f : ex2(s[j] - m_use);
        const float p1 = s[j + 1] == -INFINITY ? 0.f : ex2(s[j + 1] - m_use);
        if constexpr (kFp8) {
          pk[j / 2] = pack_bf16x2(p0 * rsc[j], p1 * rsc[j + 1]);
          lsum += p0 + p1;
        } else {
          const uint32_t w = pack_bf16x2(p0, p1);
          pk[j / 2] = w;
          lsum += p0 + p1;
          lsum_pv += __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
        }
      }
      // P buffer and O are free once PV(i-1) has completed
      const bool f2 = i >= 1 ? !mbar_wait(BAR(BAR_PVD), (i - 1) & 1) : false;
      if (group_any(f2, 2, 128)) { aborted = true; break; }
      tc_fence_after();
      const bool resc = need && i >= 1 && m_run > -INFINITY;
      if (group_any(resc, 2, 128)) {
        if (half == 0) s_alpha[h] = resc ? alpha : 1.f;
        named_bar_sync(2, 128);
        // O^T lanes are dims, columns are heads: scale column k by alpha[k]
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_base + kColO + 32u * (uint32_t)c;
          tmem_ld_32x32b_x32(ta, o);
          tmem_wait_ld();
          const float* al = s_alpha + (c & 1) * 32;
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= al[k];
          tmem_st_32x32b_x32(ta, o);
        }
        tmem_wait_st();
      }
      l_run = l_run * alpha + lsum;
      l_pv = kFp8 ? l_run : l_pv * alpha + lsum_pv;
      m_run = m_use;
      const uint32_t prow = sbase + kSmemP;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        st_shared_v4(prow + sw128_off(h, half * 4 + q4),
                     make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(BAR_PF));
    }
    // ---------------------------------------------------------- epilogue
    if (!aborted && ntiles > 0) {
      const bool f = !mbar_wait(BAR(BAR_PVD), (ntiles - 1) & 1);
      aborted = group_any(f, 2, 128);
      tc_fence_after();
    }
    if (!aborted) {
      const float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      const float l_nrm = l_pv + __shfl_xor_sync(0xffffffffu, l_pv, 16);
      const bool any = l_tot > 0.f;
      if (half == 0) {
        s_invl[h] = any ? 1.f / l_nrm : 0.f;
        s_lse[h] = any ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
      }
      named_bar_sync(2, 128);
      const bool direct = p.nsplit == 1;
      // stage [64 heads][512 dims] in the (now idle) KV buffers
      __nv_bfloat16* st_bf = reinterpret_cast<__nv_bfloat16*>(smem + kSmemKV);
      float* st_f = reinterpret_cast<float*>(smem + kSmemKV);
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        float o[32];
        if (ntiles > 0) {
          tmem_ld_32x32b_x32(tmem + lane_base + kColO + 32u * (uint32_t)c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0.f;
        }
        const int dim = (c >> 1) * 128 + 32 * warp + lane;
        const int h0 = (c & 1) * 32;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float val = o[k] * s_invl[h0 + k];
          if (direct) st_bf[(h0 + k) * kDv + dim] = __float2bfloat16_rn(val);
          else st_f[(h0 + k) * kDv + dim] = val;
        }
      }
      named_bar_sync(2, 128);
      const int tid = threadIdx.x;  // 0..127
      if (direct) {
        const uint4* src = reinterpret_cast<const uint4*>(st_bf);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)b * kH * kDv);
        for (int i = tid; i < kH * kDv * 2 / 16; i += 128) dst[i] = src[i];
        if (half == 0) p.lse[(size_t)b * kH + h] = s_lse[h];
      } else {
        const size_t part = (size_t)b * p.nsplit + split;
        const uint4* src = reinterpret_cast<const uint4*>(st_f);
        uint4* dst = reinterpret_cast<uint4*>(p.part_o + part * kH * kDv);
        for (int i = tid; i < kH * kDv * 4 / 16; i += 128) dst[i] = src[i];
        if (half == 0) p.part_lse[part * kH + h] = s_lse[h];
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================ combine kernel
// One block per (head, sequence); 128 threads x 4 dims.
__global__ void __launch_bounds__(128) smla_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           __nv_bfloat16* __restrict__ out,
                                                           float* __restrict__ lse, int nsplit) {
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const float* pl = part_lse + (size_t)b * nsplit * kH + h;
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, pl[(size_t)s * kH]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = -INFINITY;
  if (mx > -INFINITY) {
    float tot = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = pl[(size_t)s * kH];
      if (ls == -INFINITY) continue;
      const float w = exp2f((ls - mx) * 1.4426950408889634f);
      tot += w;
      const float4 o = reinterpret_cast<const float4*>(part_o + (((size_t)b * nsplit + s) * kH + h) * kDv)[t];
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
    const float inv = 1.f / tot;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    L = mx + logf(tot);
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  reinterpret_cast<uint2*>(out + ((size_t)b * kH + h) * kDv)[t] = pk;
  if (t == 0) lse[(size_t)b * kH + h] = L;
}

// ============================================================ host side
static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static smla_status validate_shape(const smla_shape* s) {
  if (!s) return SMLA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535 || s->topk < 1 || s->topk > (1 << 24)) return SMLA_ERR_INVALID_ARG;
  if (s->num_kv_rows < 1 || s->num_kv_rows > 0x7FFFFFFFLL) return SMLA_ERR_INVALID_ARG;
  if (s->nsplit < 0 || s->reserved != 0) return SMLA_ERR_INVALID_ARG;
  if (s->num_heads != kH || s->d_qk != kDqk || s->d_v != kDv) return SMLA_ERR_UNSUPPORTED;
  if (s->kv_dtype != SMLA_KV_BF16 && s->kv_dtype != SMLA_KV_FP8_E4M3_ROWSCALE) return SMLA_ERR_UNSUPPORTED;
  if (s->page_size != 0 && s->page_size != 64) return SMLA_ERR_UNSUPPORTED;
  if (s->page_size != 0 && s->pages_per_seq < 1) return SMLA_ERR_INVALID_ARG;
  return SMLA_OK;
}

static int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = n;
  return n;
}

static int plan_nsplit(const smla_shape* s, int num_sms) {
  const int tiles = (s->topk + kTile - 1) / kTile;
  int n;
  if (s->nsplit > 0) {
    n = s->nsplit;
  } else {
    n = num_sms > 0 ? num_sms / s->batch : 1;
  }
  if (n < 1) n = 1;
  if (n > tiles) n = tiles;
  return n;
}

static size_t partial_bytes(int batch, int nsplit) {
  const size_t o = (size_t)batch * nsplit * kH * kDv * 4;
  const size_t l = (size_t)batch * nsplit * kH * 4;
  return ((o + l + 255) / 256) * 256;
}

// The shared-memory opt-in is set once per device (an idempotent call, so a
// race between threads is harmless); later calls, including calls made
// while a stream is being captured into a CUDA graph, skip it.
template <bool kFp8>
static cudaError_t ensure_smem_attr() {
  static volatile int done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(smla_split_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
  return e;
}

template <bool kFp8>
static cudaError_t launch_split(const SplitParams& prm, cudaStream_t stream) {
  auto kern = smla_split_kernel<kFp8>;
  cudaError_t e = ensure_smem_attr<kFp8>();
  if (e != cudaSuccess) return e;
  dim3 grid(prm.nsplit, prm.batch);
  kern<<<grid, Cfg<kFp8>::kThreads, kSmemBytes, stream>>>(prm);
  return cudaGetLastError();
}

static smla_status run_split(const smla_shape* shape, const void* q, const void* kv_cache,
                             const float* kv_row_scale, const int32_t* page_table, const int32_t* indices,
                             float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                             int32_t* nsplit_out, cudaStream_t stream, int* nsplit_used) {
  smla_status st = validate_shape(shape);
  if (st != SMLA_OK) return st;
  if (!q || !kv_cache || !indices || !out || !lse) return SMLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16) || !aligned(indices, 4) || !aligned(lse, 4))
    return SMLA_ERR_INVALID_ARG;
  const bool fp8 = shape->kv_dtype == SMLA_KV_FP8_E4M3_ROWSCALE;
  if (fp8 && (!kv_row_scale || !aligned(kv_row_scale, 4))) return SMLA_ERR_INVALID_ARG;
  if (shape->page_size && (!page_table || !aligned(page_table, 4))) return SMLA_ERR_INVALID_ARG;
  if (!(scale == scale) || isinf(scale)) return SMLA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return SMLA_ERR_CUDA;
  const int n = plan_nsplit(shape, sms);
  if (n > 1) {
    if (!workspace || !aligned(workspace, 256)) return SMLA_ERR_WORKSPACE;
    if (workspace_bytes < partial_bytes(shape->batch, n)) return SMLA_ERR_WORKSPACE;
  }
  SplitParams prm;
  prm.q = static_cast<const uint8_t*>(q);
  prm.kv = static_cast<const uint8_t*>(kv_cache);
  prm.kv_row_scale = kv_row_scale;
  prm.page_table = page_table;
  prm.indices = indices;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.part_o = static_cast<float*>(workspace);
  prm.part_lse = n > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                  (size_t)shape->batch * n * kH * kDv * 4)
                       : nullptr;
  prm.batch = shape->batch;
  prm.topk = shape->topk;
  prm.nsplit = n;
  prm.ntiles_total = (shape->topk + kTile - 1) / kTile;
  prm.page_size = shape->page_size;
  prm.pages_per_seq = shape->pages_per_seq;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
  const cudaError_t e = fp8 ? launch_split<true>(prm, stream) : launch_split<false>(prm, stream);
  if (e != cudaSuccess) return SMLA_ERR_CUDA;
  if (nsplit_out) *nsplit_out = n;
  if (nsplit_used) *nsplit_used = n;
  return SMLA_OK;
}

static smla_status run_combine(int batch, int nsplit, const float* part_o, const float* part_lse, void* out,
                               float* lse, cudaStream_t stream) {
  dim3 grid(kH, batch);
  smla_combine_kernel<<<grid, 128, 0, stream>>>(part_o, part_lse, static_cast<__nv_bfloat16*>(out), lse, nsplit);
  return cudaGetLastError() == cudaSuccess ? SMLA_OK : SMLA_ERR_CUDA;
}

}  // namespace smla

// ============================================================ C ABI
extern "C" {

int32_t sparse_mla_abi_version(void) { return SMLA_ABI_VERSION; }

const char* sparse_mla_status_string(smla_status s) {
  switch (s) {
    case SMLA_OK: return "SMLA_OK";
    case SMLA_ERR_INVALID_ARG: return "SMLA_ERR_INVALID_ARG";
    case SMLA_ERR_UNSUPPORTED: return "SMLA_ERR_UNSUPPORTED";
    case SMLA_ERR_WORKSPACE: return "SMLA_ERR_WORKSPACE";
    case SMLA_ERR_CUDA: return "SMLA_ERR_CUDA";
    case SMLA_ERR_DEVICE_TIMEOUT: return "SMLA_ERR_DEVICE_TIMEOUT";
  }
  return "SMLA_ERR_UNKNOWN";
}

int32_t sparse_mla_plan_nsplit(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return 0;
  return smla::plan_nsplit(shape, smla::device_sm_count());
}

size_t sparse_mla_workspace_size(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return 0;
  const int n = smla::plan_nsplit(shape, smla::device_sm_count());
  return n > 1 ? smla::partial_bytes(shape->batch, n) : 0;
}

smla_status sparse_mla_decode_split(const smla_shape* shape, const void* q, const void* kv_cache,
                                    const float* kv_row_scale, const int32_t* page_table,
                                    const int32_t* indices, float scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, int32_t* nsplit_out,
                                    void* stream) {
  return smla::run_split(shape, q, kv_cache, kv_row_scale, page_table, indices, scale, out, lse, workspace,
                         workspace_bytes, nsplit_out, static_cast<cudaStream_t>(stream), nullptr);
}

smla_status sparse_mla_decode(const smla_shape* shape, const void* q, const void* kv_cache,
                              const float* kv_row_scale, const int32_t* page_table, const int32_t* indices,
                              float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream) {
  int n = 0;
  const smla_status st = smla::run_split(shape, q, kv_cache, kv_row_scale, page_table, indices, scale, out, lse,
                                         workspace, workspace_bytes, nullptr, static_cast<cudaStream_t>(stream),
                                         &n);
  if (st != SMLA_OK || n == 1) return st;
  const float* po = static_cast<const float*>(workspace);
  const float* pl = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) +
                                                   (size_t)shape->batch * n * smla::kH * smla::kDv * 4);
  return smla::run_combine(shape->batch, n, po, pl, out, lse, static_cast<cudaStream_t>(stream));
}

smla_status sparse_mla_combine(int32_t batch, int32_t num_heads, int32_t d_v, int32_t nsplit,
                               const float* partial_o, const float* partial_lse, void* out, float* lse,
                               void* stream) {
  if (batch < 1 || batch > 65535 || nsplit < 1 || nsplit > 4096) return SMLA_ERR_INVALID_ARG;
  if (num_heads != smla::kH || d_v != smla::kDv) return SMLA_ERR_UNSUPPORTED;
  if (!partial_o || !partial_lse || !out || !lse) return SMLA_ERR_INVALID_ARG;
  if (!smla::aligned(partial_o, 16) || !smla::aligned(out, 16) || !smla::aligned(partial_lse, 4) ||
      !smla::aligned(lse, 4))
    return SMLA_ERR_INVALID_ARG;
  return smla::run_combine(batch, nsplit, partial_o, partial_lse, out, lse, static_cast<cudaStream_t>(stream));
}

smla_status sparse_mla_get_device_error(uint32_t* code) {
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, smla::g_error_word, sizeof(w)) != cudaSuccess) return SMLA_ERR_CUDA;
  const unsigned int zero = 0;
  if (w != 0 && cudaMemcpyToSymbol(smla::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SMLA_ERR_CUDA;
  if (code) *code = w;
  return w ? SMLA_ERR_DEVICE_TIMEOUT : SMLA_OK;
}

}  // extern "C"
