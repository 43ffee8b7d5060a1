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
//    (decode row, top-k chunk); 64-token tiles are gathered into shared
//    memory with 16-byte cp.async and consumed by the tensor cores for every
//    head (fp8 rows as stored; DeepSeek-V4 pages through convert warps).
//  * Scores and PV as tensor-core contractions across the head group with
//    fp32 accumulation ([Design] "Design Decisions" 5-6).  Here: tcgen05.mma
//    with accumulators in tensor memory (TMEM):
//        S  = Q . K^T   M = 64 heads, N = 64 tokens, K = 576, Q read from TMEM
//        O += P . V     M = 64 heads, N = 2 x 256 dims, K = 64 tokens
//    (kind::f16 for bf16 rows; kind::f8f6f4 on the fp8 codes, with the
//    query and P as exact e4m3 high + low parts).  The query sits in tensor
//    memory and several 64-row tiles in shared memory: B200's 227 KB per CTA
//    lets BLOCK_H = 64 (all heads) fit, which the pages' ~99 KB sm_120
//    budget forbade ([Design] "Memory Budgeting").
//  * Online softmax in fp32; masked entries (index -1) take no part
//    ([Design] "Edge Case Handling").  Rows of masked entries are zero-filled
//    in shared memory and their probabilities are exactly 0.
//  * Split-K over the top-k list with a log-sum-exp combine, so that small
//    batches still spread over all SMs; the split count is a pure function of
//    (batch, top-k, SM count) so that the grid is fixed per batch bucket for
//    CUDA-graph capture ([Truth] "The Split-K Solution: Reasoning About the
//    Fix"; [Pivot] "The Reasoning: Weighing Two Paths").
//
// Warp roles in the split kernel (one CTA per SM; ~223-227 KB shared
// memory), set per cache kind by Cfg below: softmax + epilogue warps (two per
// TMEM lane quarter; one for DeepSeek-V4 pages), the MMA issuers (S and PV;
// fp8: four, one per SM sub-partition), the index resolvers, the copy warps
// and, for DeepSeek-V4 pages, the convert warps.
// Every wait on a pipeline barrier is bounded (about 2 s): on expiry the CTA
// records an error bit in a device word, drains its own copies and MMAs,
// frees TMEM and exits.

#include <cuda.h>            // CUtensorMap (the indexer's key loads)
#include <cudaTypedefs.h>    // PFN_cuTensorMapEncodeTiled
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

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

constexpr int kRawRowBytes = 576;                   // fp8 row / DeepSeek-V4 slot (codes as stored)
constexpr int kRawTileBytes = kTile * kRawRowBytes; // 36,864

// Shared memory map (offsets from the 1024-aligned dynamic shared base):
//   [operand stages][raw stages][aux]
// Operand stage: one 64-row tile as bf16, 9 atoms of [64 rows][128 B],
// 128-byte swizzled (K-major for S, MN-major for PV).  P(t) [64 heads][64
// tok] bf16 (K-major) takes the place of the rope atom of the stage that
// holds tile t: S(t) has read that atom by the time P(t) is written, PV(t)
// reads the rest of the stage, and the stage is refilled only after PV(t).
// Each stage thus carries its own P buffer.
// Raw stage (DeepSeek-V4 caches): one tile's rows as stored, 576
// contiguous bytes per row, before conversion to bf16.
// fp8 caches compute on the codes as stored: an operand stage is one tile
// of 576-code rows as 8-row x 16-byte core matrices (no swizzle; K-major
// for S, MN-major for PV), and P(t) goes to one of four separate P buffers
// ([64 heads][128 codes: 64 tokens high part, 64 low part], 128-byte
// swizzled, K-major).
constexpr int kSmemKV = 0;
constexpr int kAtomP = kAtoms - 1;
constexpr int kRing = 4;                            // resolved-row ring depth (tiles)
constexpr int kMaxStages = 5;
constexpr int kNumS = 3;                            // S buffers in tensor memory
constexpr int kMaxPieces = 3;                       // stream-K: CTAs that may share one row (rows > G / 2)
// barrier indices
constexpr int BAR_KVF = 0;                          // [stages] operand tile ready
constexpr int BAR_KVE = BAR_KVF + kMaxStages;       // [stages] operand tile consumed (PV done)
constexpr int BAR_SF = BAR_KVE + kMaxStages;        // [kNumS] S(t) in TMEM
constexpr int BAR_SE = BAR_SF + kNumS;              // [kNumS] S(t) read by the softmax
constexpr int BAR_PF = BAR_SE + kNumS;              // [stages] P(t) written (per stage)
constexpr int BAR_PVD = BAR_PF + kMaxStages;        // [4] PV(t) done (by t mod 4)
constexpr int BAR_FIN = BAR_PVD + 4;                // drain, S issuer
constexpr int BAR_FIN2 = BAR_FIN + 1;               // drain, PV issuer
constexpr int BAR_QT = BAR_FIN2 + 1;                // query written to TMEM
constexpr int BAR_QS = BAR_QT + 1;                  // query staged in shared memory
constexpr int BAR_IXF = BAR_QS + 1;                 // [kRing] rows resolved
constexpr int BAR_IXS = BAR_IXF + kRing;            // [kRing] row scales / scale blocks resolved
constexpr int BAR_IXE = BAR_IXS + kRing;            // [kRing] rows consumed
constexpr int BAR_RAW = BAR_IXE + kRing;            // [raw stages] raw rows landed
constexpr int BAR_RAWE = BAR_RAW + kMaxStages;      // [raw stages] raw rows converted
constexpr int BAR_CS1 = BAR_RAWE + kMaxStages;      // cluster: every split's blocks written
constexpr int BAR_SH = BAR_CS1 + 1;                 // [kNumS] S(t) high part done (split S issue)
constexpr int BAR_FIN3 = BAR_SH + kNumS;            // drain, second S issuer
constexpr int BAR_FIN4 = BAR_FIN3 + 1;              // drain, second PV issuer
constexpr int kNumBars = BAR_FIN4 + 1;
// DeepSeek-V4 page: 64 slots of 576 bytes (448 e4m3fn codes, 64 bf16), then
// 64 scale blocks of 8 bytes (7 UE8M0 exponents, one per 64 code dims)
constexpr int kDsv4Slot = 576, kDsv4Nope = 448;
constexpr int kDsv4ScaleOff = 64 * kDsv4Slot;       // 36,864
constexpr int kDsv4Page = kDsv4ScaleOff + 64 * 8;   // 37,376

// Tensor memory (512 columns x 128 lanes).  Each warp quarter (32 lanes)
// holds 16 heads; an M=64 operand or accumulator uses lanes 0-15 or 16-31
// of every quarter.
//   lanes 0-15 : Q (A operand of S, bf16 packed two per column) cols [0,288)
//                S buffers (fp32, 64 columns each)         cols [288,480)
//   lanes 16-31: O (fp32, 64 heads x 512 dims)             cols [0,512)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS = 288;
constexpr uint32_t kLaneO = 16;
static_assert(kColS + 64u * kNumS <= kTmemCols, "S buffers fit beside the query");

// Lazy rescaling: keep the running max until a new max exceeds it by more
// than 2^8 (probabilities stay <= 256; results are unchanged).
constexpr float kRescaleThresh = 8.0f;

// Instruction descriptors (kind::f16): D f32 (bits 4-5 = 1), A bf16 (7-9 = 1),
// B bf16 (10-12 = 1), A major bit 15, B major bit 16, N>>3 at 17, M>>4 at 24.
constexpr uint32_t make_idesc(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescS = make_idesc(64, 64, false, false);    // S = Q K^T   (Q from TMEM)
constexpr uint32_t kIdescPV = make_idesc(64, 256, false, true);   // O += P V    (V MN-major)
// Instruction descriptors (kind::f8f6f4): D f32, A and B e4m3 (format 0 in
// bits 7-9 and 10-12), B major bit 16, N>>3 at 17, M>>4 at 24.
constexpr uint32_t make_idesc_e4m3(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescS8 = make_idesc_e4m3(64, 64, false);    // S = [Qhi | Qlo] [K; K]^T
constexpr uint32_t kIdescPV8 = make_idesc_e4m3(64, 256, true);   // O += [Phi | Plo] [V; V]

// Bounded waits give up after this many SM clock cycles (about 2 s).
constexpr long long kWaitLimitCycles = 4000000000ll;

// Warp roles: S softmax/epilogue warps (two per tensor-memory lane quarter,
// or one for DeepSeek-V4 caches), then the S-MMA issuer (+ TMEM allocator),
// the PV-MMA issuer, the index resolvers (four, or two for fp8 rows:
// resolver k owns the tiles t = k mod their count), the copy warps and, for
// DeepSeek-V4 caches, eight warps that convert the raw codes to bf16 operand
// tiles.  The in-cluster merge uses warps 0-7 and, for the lse, warps 8-9,
// all done with their roles by then.
// cache layouts the split kernel is instantiated for
constexpr int kKindBf16 = 0;   // bf16 rows [N, 576]
constexpr int kKindFp8 = 1;    // e4m3fn rows [N, 576] + one fp32 scale per row
constexpr int kKindDsv4 = 2;   // DeepSeek-V4 pages: 448 e4m3fn + UE8M0 group scales, 64 bf16 rope
template <int kKind>
struct Cfg {
  static constexpr bool kNat = kKind == kKindFp8;       // e4m3 MMAs on the codes as stored
  static constexpr bool kConv = kKind == kKindDsv4;     // raw codes converted to bf16 by convert warps
  static constexpr int kStages = kNat ? 5 : (kConv ? 2 : 3);   // operand stages
  static constexpr int kOpBytes = kNat ? kRawTileBytes : kTileBytes;   // bytes per operand stage
  static constexpr int kRawStages = kConv ? 2 : 0;      // raw stages
  // the staged query (64 x d_qk bf16) sits in the last operand stage (bf16
  // operands), or the last two (fp8: 73,728 B = two 36,864 B stages) until
  // it is in TMEM
  static constexpr int kQStage = kNat ? kStages - 2 : kStages - 1;
  static constexpr int kSmxWarps = kConv ? 4 : 8;
  // MMA issuers.  fp8: four, one per SM sub-partition (warp w runs on
  // sub-partition w mod 4): S(t) is issued in two halves, the query's high
  // part by kWarpS and then, once that has completed, its low part by
  // kWarpS2 (18 MMAs each), and PV(t) by kWarpPV (dims 0-255) and kWarpPV2
  // (256-511).  A warp issuing a long run of MMAs slows the softmax warps
  // of its own sub-partition, which then hold up every PV; spread over the
  // four sub-partitions this measured faster than two issuers (c5: 73.4 ->
  // 68.0 us).  With two copy warps (below) each sub-partition holds two
  // softmax warps, one issuer and an index or a copy warp; the S halves
  // beside the index warps (warps 8, 9) and the PV halves beside the copy
  // warps (10, 11) measured best of the placements tried.
  static constexpr bool kSplitIss = kNat;
  static constexpr int kWarpS = kSmxWarps, kWarpPV = kSmxWarps + (kSplitIss ? 2 : 1);
  static constexpr int kWarpS2 = kSplitIss ? kSmxWarps + 1 : -1, kWarpPV2 = kSplitIss ? kSmxWarps + 3 : -1;
  static constexpr int kWarpIdx = kSmxWarps + (kSplitIss ? 4 : 2);
  // fp8: two resolvers (16 warps in all, 128 registers a thread) measured
  // ~2 % faster on 2048-entry lists; bf16 operands keep four (two were ~4 %
  // slower on 512-entry lists)
  static constexpr int kIdxWarps = kNat ? 2 : 4;
  static constexpr int kWarpLoad0 = kWarpIdx + kIdxWarps;
  // copy warps: fp8 rows two (16 warps in all, four per sub-partition:
  // c5 66.7 -> 62.7 us against four), bf16 rows four
  static constexpr int kCopyWarps = kConv || kNat ? 2 : 4;
  static constexpr int kCvtWarps = kConv ? 8 : 0;
  static constexpr int kCopyThreads = kCopyWarps * 32;
  static constexpr int kLoadWarps = kCopyWarps + kCvtWarps;
  static constexpr int kThreads = (kWarpLoad0 + kLoadWarps) * 32;
  // Raw tiles: 8-row groups g < kCpGroups arrive by 16-byte cp.async, the
  // rest by one bulk copy per row (the copy engine adds bandwidth to the
  // load/store path's); copy warp w owns the groups g = w mod kCopyWarps.
  static constexpr int kCpGroups = kConv ? 5 : 8;
  static constexpr int kBulkGroups = 8 - kCpGroups;      // one expect-tx arrival each
  // shared memory map
  static constexpr int kSmemP = kSmemKV + kStages * kOpBytes;             // fp8: four P buffers
  static constexpr int kSmemRaw = kSmemP + (kNat ? 4 * kAtomBytes : 0);
  static constexpr int kSmemAux = kSmemRaw + kRawStages * kRawTileBytes;
  static constexpr int kAuxBars = kSmemAux;
  static constexpr int kAuxTmem = (kAuxBars + 8 * kNumBars + 15) / 16 * 16;  // TMEM base address (4 B)
  static constexpr int kAuxRow = kAuxTmem + 16;              // int  [kRing][64] physical row or -1
  static constexpr int kAuxRsc = kAuxRow + kRing * 64 * 4;   // f32  [kRing][64] fp8 row scales
  static constexpr int kAuxDsc = kAuxRsc + kRing * 64 * 4;   // u64  [kRing][64] DeepSeek-V4 scale blocks
  static constexpr int kAuxXch = kAuxDsc + kRing * 64 * 8;   // f32  [2][2][64] softmax exchange
  static constexpr int kAuxQsc = kAuxXch + 2 * 2 * 64 * 4;   // f32  [64] fp8 query scales
  static constexpr int kAuxFlag = kAuxQsc + 64 * 4;          // int  [4] stream-K: last piece of the row (per quarter)
  static constexpr int kSmemBytes = kAuxFlag + 4 * 4;
  static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-CTA shared memory of sm_100");
  static_assert(kAuxRow % 16 == 0 && kAuxRsc % 16 == 0 && kAuxDsc % 16 == 0, "aux arrays are read as vectors");
  static_assert(8 % kCopyWarps == 0 && kCpGroups >= 1 && kCpGroups <= 8, "copy-warp group ownership");
  static_assert(!kConv || kCvtWarps == 8, "convert warps: one thread per (row, 16-code column)");
  static_assert(kSmemP % 1024 == 0, "P buffers are 128-byte swizzled (1024-byte aligned)");
  static_assert(kStages <= kMaxStages, "barrier arrays");
  static_assert(kSmxWarps == 4 || kSmxWarps == 8, "one or two softmax warps per lane quarter");
  static_assert(kWarpLoad0 >= 10, "warps 8 and 9 exist beside the merging warps 0-7");
};

struct SplitParams {
  const uint8_t* q;            // [B, 64, 576] bf16
  const uint8_t* kv;           // rows of 1152 B (bf16) or 576 B (fp8 codes)
  const float* kv_row_scale;   // [N] (fp8)
  const int32_t* page_table;   // [B, pages_per_seq] (paged)
  const int32_t* indices;      // [B, topk]
  __nv_bfloat16* out;          // [B, 64, 512]
  float* lse;                  // [B, 64]
  float* part_o;               // [B, nsplit, 64, 512]; stream-K: [2 G, 64, 512] piece results
  float* part_lse;             // [B, nsplit, 64]; stream-K: [2 G, 64] their lse (log2 units)
  unsigned long long* row_ctr; // stream-K: [B, 4] arrivals per (row, lane quarter), tagged with epoch
  unsigned long long epoch;    // stream-K: this launch's tag (1 .. 2^56 - 1)
  int streamk;                 // 1: the G CTAs of the grid share the rows' tiles evenly (stream-K)
  int batch, topk, nsplit, ntiles_total;   // batch: decode rows (sequences x tokens)
  int tok_per_seq;             // query tokens per sequence (row b reads page-table row b / tok_per_seq)
  int cluster;                 // 1: the nsplit CTAs of a sequence form a cluster and reduce on chip
  int page_size, pages_per_seq;
  int num_kv_rows;             // rows in the pool (64 x pages when paged)
  float scale_log2;            // scale * log2(e)
  long long wait_limit;        // cycles a pipeline wait may take before it gives up
  int stall_test;              // 1: the score issuer waits on a barrier nothing arrives on (test of the bounded waits)
};

__device__ unsigned int g_error_word = 0;

// Scratch for sparse_mla_decode_static_scratch: split partials for callers
// that cannot allocate (one buffer per device, shared by all such calls).
static __device__ __align__(256) unsigned char g_static_scratch[SMLA_STATIC_SCRATCH_BYTES];

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
// Bounded wait: false (and an error bit) if the phase did not complete
// within `limit` SM clock cycles.  The first probe is inline; the loop is
// out of line.
__device__ __noinline__ bool mbar_wait_loop(uint32_t bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit) {
      atomicOr(&g_error_word, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit = kWaitLimitCycles) {
  return mbar_try_wait(bar, parity) || mbar_wait_loop(bar, parity, limit);
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
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// two fp32 -> packed f16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// two fp32 -> packed bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// bf16x2 product, round to nearest even
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Four fp8 e4m3fn codes (one 32-bit word, lowest byte first) -> two packed
// bf16x2 words (codes 0,1 and 2,3), exact for every non-NaN code, with
// integer and bf16x2 arithmetic only (the conversion instructions run at a
// fraction of that rate).  Each code's sign goes to bit 15 and its exponent
// and mantissa bits to bits 10..4 of a bf16, which then holds the code's
// value times 2^-120: the exponent field is read with bias 127 instead of 7,
// and a zero exponent field reads as a bf16 subnormal just as it reads as an
// e4m3 subnormal.  One bf16 multiply by 2^120 (subnormal inputs are kept,
// the product is exact) restores the value.  NaN codes come out finite.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  constexpr uint32_t kTwo120 = 0x7B807B80u;          // 2^120 in both bf16 halves
  const uint32_t u0 = __byte_perm(w, 0, 0x4140);     // code 1 -> bits 23..16, code 0 -> bits 7..0
  const uint32_t u1 = __byte_perm(w, 0, 0x4342);     // codes 3, 2
  // (sign << 15) | (magnitude << 4) per half: 16 u + 240 (u & signs)
  const uint32_t b0 = u0 * 16u + (u0 & 0x00800080u) * 240u;
  const uint32_t b1 = u1 * 16u + (u1 & 0x00800080u) * 240u;
  lo = bf16x2_mul(b0, kTwo120);
  hi = bf16x2_mul(b1, kTwo120);
}
// The same, times a power of two given as a bf16x2 pair s2 (both halves
// equal): the exact code value first, then one more rounding multiply,
// exact whenever the product is a bf16 normal number.
__device__ __forceinline__ void e4m3x4_to_bf16x4_scaled(uint32_t w, uint32_t s2, uint32_t& lo, uint32_t& hi) {
  e4m3x4_to_bf16x4(w, lo, hi);
  lo = bf16x2_mul(lo, s2);
  hi = bf16x2_mul(hi, s2);
}
// Two fp32 -> packed e4m3x2 (lo in the low byte), round to nearest even,
// saturating at +-448.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// packed e4m3x2 (low byte first) -> two fp32, exact
__device__ __forceinline__ float2 unpack_e4m3x2(uint32_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)v));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
// x = hi + lo with hi = e4m3(x) and lo = e4m3(x - hi): exact for a bf16 x
// (8 significant bits) whose parts are e4m3 normals, and within half an
// e4m3 subnormal step (2^-10) otherwise.  Returns hi and lo as e4m3x2
// pairs for (x0, x1).
__device__ __forceinline__ void split_e4m3x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_e4m3x2(x0, x1);
  const float2 h = unpack_e4m3x2(hi);
  lo = pack_e4m3x2(x0 - h.x, x1 - h.y);
}
// The same split through f16x2: x is rounded to f16 first (11 significant
// bits, relative error <= 2^-12), then hi = e4m3(x16), lo = e4m3(x16 - hi)
// (the difference is exact in f16).  For x in [0, 448).
__device__ __forceinline__ void split_e4m3x2_h(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const uint32_t x16 = pack_f16x2(x0, x1);
  uint16_t h, l;
  uint32_t h16, r16;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(h) : "r"(x16));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h16) : "h"(h));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r16) : "r"(x16), "r"(h16));
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(l) : "r"(r16));
  hi = h;
  lo = l;
}
// 2^k for an integer k in [-126, 127]
__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }
// floor(log2(x)) for a normal positive x
__device__ __forceinline__ int ilog2f(float x) { return (int)((__float_as_uint(x) >> 23) & 0xFFu) - 127; }
// UE8M0 exponent byte e (OCP microscaling E8M0) -> 2^(e - 127) as a bf16x2
// pair: the byte is the bf16 exponent field, except e = 0 (2^-127, a bf16
// subnormal) and e = 255 (E8M0 NaN; reads as infinity here).
__device__ __forceinline__ uint32_t ue8m0_bf16x2(uint32_t e) {
  const uint32_t h = e ? (e << 7) : 0x40u;
  return h | (h << 16);
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
// Warp-uniform MMA issue: the whole warp computes the (uniform) operands and
// one elected lane executes the instruction.  D[tmem] = A . B ("set", first K
// step) or D[tmem] += A . B ("acc").
__device__ __forceinline__ void mma_set_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.u32 p, 0, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_acc_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.eq.u32 p, 0, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc)
      : "memory");
}
// Same with the A operand read from tensor memory (K-major): D = A[tmem] . B
__device__ __forceinline__ void mma_ts_set_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.u32 p, 0, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_ts_acc_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.eq.u32 p, 0, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc)
      : "memory");
}
// kind::f8f6f4 (e4m3 x e4m3, fp32 accumulate): A from tensor memory (S) or
// shared memory (PV)
__device__ __forceinline__ void mma8_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              bool acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.u32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}
__device__ __forceinline__ void mma8_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              bool acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.u32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}
__device__ __forceinline__ void commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
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
// 16 lanes x 16 columns, twice: threads 0-15 read columns [c, c+16) of
// lanes base+0..15, threads 16-31 read columns [c+32, c+48) of the same lanes.
__device__ __forceinline__ void tmem_ld_16x32bx2_x16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 lanes x 32 columns, twice: threads 0-15 access columns [c, c+32) of
// lanes base+0..15, threads 16-31 columns [c+256, c+288) of the same lanes.
__device__ __forceinline__ void tmem_ld_16x32bx2_x32_h256(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 256;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st_16x32bx2_x32_h256(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 256, "
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
// 16 lanes x 16 columns, twice: threads 0-15 write columns [c, c+16) of
// lanes base+0..15, threads 16-31 columns [c+144, c+160) (the query's second
// 288 dims).
// kSplit: column offset of the second half (lanes 16-31 of the warp)
template <int kSplit>
__device__ __forceinline__ void tmem_st_16x32bx2_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %17, "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "n"(kSplit)
      : "memory");
}

// 16 lanes x 8 columns, twice: threads 0-15 write columns [c, c+8) of lanes
// base+0..15, threads 16-31 columns [c+kSplit, c+kSplit+8).
template <int kSplit>
__device__ __forceinline__ void tmem_st_16x32bx2_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], %9, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
      "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "n"(kSplit)
      : "memory");
}

// Shared-memory matrix descriptor without swizzle (layout type 0): 8-row x
// 16-byte core matrices of 128 contiguous bytes.  K-major operand: lbo =
// the next 16 bytes along K, sbo = the next 8 rows; MN-major operand: lbo
// = the next 8 rows along K, sbo = the next 16 bytes along MN.
__device__ __forceinline__ uint64_t cm_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// byte offset of 16-byte chunk c (0..35) of row r in a tile of 576-byte
// rows held as core matrices: [8-row group][chunk][row in group][16 B]
__device__ __forceinline__ uint32_t cm_off(int r, int c) {
  return (uint32_t)(((r >> 3) * (kRawRowBytes / 16) + c) * 128 + (r & 7) * 16);
}
constexpr uint32_t kCmGroupBytes = (kRawRowBytes / 16) * 128;   // 4,608: next 8 rows

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

__device__ __forceinline__ void bulk_store_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// ---- thread-block cluster (distributed shared memory)
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_shared_v4f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4f(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
// arrive (release at cluster scope) on an mbarrier of any CTA of the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with acquire at cluster scope (sees what the arriving CTAs
// released); false and an error bit on time-out.
__device__ __noinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_error_word, 1u);
      return false;
    }
  }
  return true;
}
// Programmatic dependent launch: the grid may start while the previous
// kernel of the stream is still running (its prologue overlaps that
// kernel's tail); griddepcontrol.wait blocks until every prerequisite grid
// has completed and its memory is visible, launch_dependents lets the next
// grid start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// every thread of every CTA of the cluster (executed unconditionally by all)
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// 2-D tensor copy (tile mode) global -> shared, box origin (x, y) in
// elements, completing on an mbarrier (x times the element size must be a
// multiple of 16 bytes)
__device__ __forceinline__ void tma_load_2d(uint32_t sdst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(sdst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load_g2s(uint32_t sdst, const void* gsrc, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(sdst),
               "l"(gsrc), "r"(bytes), "r"(bar)
               : "memory");
}

// Merge statistics per (split, head): m, l_pv, l, -, then the inverse fp16
// scale of each 128-dim part of the split's exchanged row.
constexpr int kStatFloats = 8;

// In-cluster merge, final step for one thread: head hh, output columns
// [col0, col0 + 128 / N) (16 / N units of 8 dims), all inside the 128-dim
// part col0 / 128.  Split s's fp16 image holds the thread's dims at lane
// hh % 16 (+16 for dims >= 256) of quarter q, unit u of the half at
// ((u / 4) * 4 + u % 4) * 32 lanes, scaled by a power of two that the
// statistics undo.  Every split's columns and statistics are loaded
// together, one L2 round trip (with 16 splits the columns follow the
// weights), then split s is weighted by 2^(m_s - M) l_pv,s and the sum
// divided by the sum of those weights.
template <int N>
__device__ __forceinline__ void merge_tail(const float* wss, const uint4* wso, int q, int lane, int hh, int col0,
                                           __nv_bfloat16* orow) {
  constexpr int kU = 16 / N;                     // units per split (16 loads in all)
  constexpr size_t kSplitU = (size_t)kH * kDv / 8;
  const uint4* src = wso + (size_t)q * (8 * 4 * 32) + (lane & 15) + 16 * (col0 >> 8);
  const int d0 = col0 & 255;
  uint4 x[16];
  auto load_columns = [&]() {
#pragma unroll
    for (int s = 0; s < N; ++s)
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int d = d0 + 8 * k;
        x[s * kU + k] = __ldcg(src + (size_t)s * kSplitU + (size_t)((d >> 5) * 4 + ((d >> 3) & 3)) * 32);
      }
  };
  // statistics [s][h][kStatFloats]; the weights need m, l_pv and the
  // inverse scale of part col0 / 128
  float w[N], lp[N], dn[N];
#pragma unroll
  for (int s = 0; s < N; ++s) {
    const float* st = wss + ((size_t)s * 64 + hh) * kStatFloats;
    const float2 v = __ldcg(reinterpret_cast<const float2*>(st));
    w[s] = v.x; lp[s] = v.y;
    dn[s] = __ldcg(st + 4 + (col0 >> 7));
  }
  // with 16 splits the columns are loaded after the weights (registers)
  if constexpr (N < 16) load_columns();
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < N; ++s) M = fmaxf(M, w[s]);
  float Lp = 0.f;
#pragma unroll
  for (int s = 0; s < N; ++s) {
    w[s] = (w[s] > -INFINITY ? ex2(w[s] - M) : 0.f) * lp[s];   // the weight of split s's normalised result
    Lp += w[s];
  }
  const float inv = Lp > 0.f ? 1.f / Lp : 0.f;
#pragma unroll
  for (int s = 0; s < N; ++s) w[s] *= dn[s];                    // undo the exchange scale
  if constexpr (N >= 16) {
    asm volatile("" ::: "memory");
    load_columns();
  }
#pragma unroll
  for (int k = 0; k < kU; ++k) {
    float a[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = 0.f;
#pragma unroll
    for (int s = 0; s < N; ++s) {
      const uint32_t w4[4] = {x[s * kU + k].x, x[s * kU + k].y, x[s * kU + k].z, x[s * kU + k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[j]));
        a[2 * j] += w[s] * f.x;
        a[2 * j + 1] += w[s] * f.y;
      }
    }
    *reinterpret_cast<uint4*>(orow + 8 * k) =
        make_uint4(pack_bf16x2(a[0] * inv, a[1] * inv), pack_bf16x2(a[2] * inv, a[3] * inv),
                   pack_bf16x2(a[4] * inv, a[5] * inv), pack_bf16x2(a[6] * inv, a[7] * inv));
  }
}

// kSK: the stream-K form (fp8 rows only), compiled apart so that the split
// plan's kernel carries none of its row switching
template <int kKind, bool kSK>
__global__ void __launch_bounds__(Cfg<kKind>::kThreads, 1)
    smla_split_kernel(const __grid_constant__ SplitParams p) {
  using C = Cfg<kKind>;
  constexpr int kCopy = C::kCopyThreads;
  constexpr bool kFp8 = kKind == kKindFp8;     // row scale folded into S and P
  constexpr bool kDsv4 = kKind == kKindDsv4;
  constexpr bool kConv = C::kConv;
  constexpr bool kNat = C::kNat;               // fp8 codes straight into e4m3 MMAs
  constexpr int kSmx = C::kSmxWarps;
  constexpr int kWarpS = C::kWarpS, kWarpPV = C::kWarpPV, kWarpIdx = C::kWarpIdx, kWarpLoad0 = C::kWarpLoad0;
  constexpr int kStages = C::kStages;
  constexpr int kQK = kDsv4 ? 512 : kDqk;      // query / key width
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kAuxBars;
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // pipeline waits give up after wl cycles (waits on copies and MMAs that
  // always complete -- the staged query, the MMA drains -- keep the default)
  const long long wl = p.wait_limit;
  const int split = blockIdx.x;
  const int nt = p.ntiles_total;                 // 64-entry tiles per decode row
  // This CTA's tiles: a run of the rows' tiles laid end to end in row order.
  // Split plan: tiles [split nt / nsplit, (split + 1) nt / nsplit) of row
  // blockIdx.y.  Stream-K plan (fp8 rows): of the W = rows x nt tiles, CTA
  // j of the G in the grid takes [j W / G, (j + 1) W / G), which can end one
  // row's run and begin the next; a row split between CTAs is merged by
  // the CTA that finishes its part last.
  constexpr bool sk = kNat && kSK;
  int b0, tr0, ntiles;                           // first tile's row and its tile within the row
  if (sk) {
    const long long W = (long long)p.batch * nt;
    const long long g0 = (long long)blockIdx.x * W / gridDim.x;
    b0 = (int)(g0 / nt);
    tr0 = (int)(g0 - (long long)b0 * nt);
    ntiles = (int)((long long)(blockIdx.x + 1) * W / gridDim.x - g0);
  } else {
    b0 = blockIdx.y;
    tr0 = (int)((long long)split * nt / p.nsplit);
    ntiles = (int)((long long)(split + 1) * nt / p.nsplit) - tr0;
  }
  const int b = b0;                              // (split plan: the row)
  // (split plan: every tile of the CTA lies in row b0)
  auto tile_row = [&](int t) -> int { return sk ? b0 + (tr0 + t) / nt : b0; };
  auto tile_in_row = [&](int t) -> int { return sk ? (tr0 + t) % nt : tr0 + t; };

  // The swizzled operand layouts need a 1024-byte aligned base; the dynamic
  // shared window starts there when the kernel has no static shared memory.
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_error_word, 2u);
    return;
  }

  int* s_row = reinterpret_cast<int*>(smem + C::kAuxRow);
  float* s_rsc = reinterpret_cast<float*>(smem + C::kAuxRsc);
  uint2* s_dsc = reinterpret_cast<uint2*>(smem + C::kAuxDsc);

  if (threadIdx.x == 0) {
    // Arrivals are per warp (the warp synchronises, one lane arrives), except
    // where a copy engine arrives: mbarrier arrivals are serialised.
    for (int s = 0; s < kStages; ++s) {
      // bf16: one arrival per copying thread (when its copies land); fp8 /
      // DeepSeek-V4: one per convert warp
      mbar_init(BAR(BAR_KVF + s), kConv ? C::kCvtWarps : kCopy);
      mbar_init(BAR(BAR_KVE + s), C::kSplitIss ? 2 : 1);   // one commit per PV issuer
      mbar_init(BAR(BAR_PF + s), kSmx);
    }
    for (int s = 0; s < C::kRawStages; ++s) {
      // one arrival per copying thread when its cp.async land, plus one
      // expect-tx arrival per 8-row group copied in bulk
      mbar_init(BAR(BAR_RAW + s), kCopy + C::kBulkGroups);
      mbar_init(BAR(BAR_RAWE + s), C::kCvtWarps);
    }
    for (int s = 0; s < kNumS; ++s) {
      mbar_init(BAR(BAR_SF + s), 1);
      mbar_init(BAR(BAR_SE + s), kSmx);
    }
    for (int s = 0; s < 4; ++s) mbar_init(BAR(BAR_PVD + s), C::kSplitIss ? 2 : 1);
    for (int s = 0; s < kNumS; ++s) mbar_init(BAR(BAR_SH + s), 1);
    mbar_init(BAR(BAR_FIN), 1);
    mbar_init(BAR(BAR_FIN2), 1);
    mbar_init(BAR(BAR_FIN3), 1);
    mbar_init(BAR(BAR_FIN4), 1);
    mbar_init(BAR(BAR_QT), 4);
    mbar_init(BAR(BAR_QS), 1);
    mbar_init(BAR(BAR_CS1), p.cluster ? p.nsplit : 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(BAR(BAR_IXF + r), 1);
      mbar_init(BAR(BAR_IXS + r), 1);
      // consumers of a ring slot: the copy warps (rows), the softmax warps
      // (row scales) and the convert warps (rows to zero, scale blocks)
      mbar_init(BAR(BAR_IXE + r), kCopy / 32 + kSmx + C::kCvtWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpS) {
    tmem_alloc(sbase + C::kAuxTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // Cluster launch: the barriers of every CTA are initialised before any
  // CTA of the cluster can arrive on them remotely.
  if (p.cluster) cluster_sync_all();
  // nothing above reads or writes global memory: with programmatic
  // dependent launch all of it overlapped the previous kernel
  grid_dep_wait();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::kAuxTmem);

  bool merge_failed = false;   // a softmax warp gave up (in-cluster merge)
  if (warp >= kWarpIdx && warp < kWarpIdx + C::kIdxWarps) {
    // ------------------------------------------------------------ index warps
    // Resolve each tile's 64 entries to physical rows (and fp8 row scales)
    // into the kRing-deep ring ahead of the loaders.  Warp k of the S =
    // kIdxWarps handles tiles t = k, k+S, ... (ring slot t mod kRing), and
    // each keeps three tiles' lookups in flight.  (Pulling the rows into L2
    // ahead of the loaders, one bulk prefetch per row, measured slower: it
    // queues on the copy engine.)
    auto idx_at = [&](int t, int j) -> int {
      if (t >= ntiles) return -1;
      const int pos = tile_in_row(t) * kTile + j;
      return pos < p.topk ? __ldg(p.indices + (size_t)tile_row(t) * p.topk + pos) : -1;
    };
    // An entry that names no row of the pool (past the page table, or a
    // row outside [0, num_kv_rows)) is read as padding and sets error bit 2.
    auto row_of = [&](int idx, int drow) -> int {   // drow: the decode row of the entry
      if (idx < 0) return -1;
      long long r = idx;
      if (p.page_size) {
        if (idx >= (long long)p.pages_per_seq * p.page_size) r = -1;
        else r = (long long)__ldg(p.page_table + (size_t)(drow / p.tok_per_seq) * p.pages_per_seq + idx / p.page_size) *
                     p.page_size +
                 idx % p.page_size;
      }
      if (r < 0 || r >= p.num_kv_rows) {
        atomicOr(&g_error_word, 4u);
        return -1;
      }
      return (int)r;
    };
    const int kw = warp - kWarpIdx;
    // the 64 x kQK query (contiguous bf16) into the last operand stage(s),
    // which no tile uses before the query has been moved to tensor memory:
    // one bulk copy
    if (kw == 0 && lane == 0) {
      constexpr uint32_t kQBytes = (uint32_t)kH * kQK * 2;
      mbar_arrive_expect_tx(BAR(BAR_QS), kQBytes);
      bulk_load_g2s(sbase + kSmemKV + C::kQStage * C::kOpBytes, p.q + (size_t)b * kQBytes, kQBytes, BAR(BAR_QS));
    }
    // Software pipeline over this warp's tiles (step S), every load
    // consumed one iteration after it was issued: index of tile t+3S, page
    // entry of t+2S, row scale of t+S, then tile t is published.
    constexpr int S = C::kIdxWarps;
    int i2_0 = idx_at(kw + 2 * S, lane), i2_1 = idx_at(kw + 2 * S, lane + 32);                 // tile t+2S
    int r1_0 = row_of(idx_at(kw + S, lane), tile_row(kw + S)),                                 // tile t+S
        r1_1 = row_of(idx_at(kw + S, lane + 32), tile_row(kw + S));
    int r0_0 = row_of(idx_at(kw, lane), tile_row(kw)), r0_1 = row_of(idx_at(kw, lane + 32), tile_row(kw));  // tile t
    float c0_0 = 0.f, c0_1 = 0.f;                                            // scale, tile t
    uint2 d0_0 = make_uint2(0u, 0u), d0_1 = make_uint2(0u, 0u);              // scale block, tile t
    // a DeepSeek-V4 row's 8-byte scale block
    auto dsc_of = [&](int r) -> uint2 {
      if (r < 0) return make_uint2(0u, 0u);
      return __ldg(reinterpret_cast<const uint2*>(p.kv + (size_t)(r >> 6) * kDsv4Page + kDsv4ScaleOff +
                                                  (r & 63) * 8));
    };
    if (kFp8) {
      c0_0 = r0_0 >= 0 ? __ldg(p.kv_row_scale + r0_0) : 0.f;
      c0_1 = r0_1 >= 0 ? __ldg(p.kv_row_scale + r0_1) : 0.f;
    }
    if (kDsv4) {
      d0_0 = dsc_of(r0_0);
      d0_1 = dsc_of(r0_1);
    }
    for (int t = kw; t < ntiles; t += S) {
      const int rs = t % kRing;
      float c1_0 = 0.f, c1_1 = 0.f;
      uint2 d1_0 = make_uint2(0u, 0u), d1_1 = make_uint2(0u, 0u);
      if (kFp8) {
        c1_0 = r1_0 >= 0 ? __ldg(p.kv_row_scale + r1_0) : 0.f;
        c1_1 = r1_1 >= 0 ? __ldg(p.kv_row_scale + r1_1) : 0.f;
      }
      if (kDsv4) {
        d1_0 = dsc_of(r1_0);
        d1_1 = dsc_of(r1_1);
      }
      const int r2_0 = row_of(i2_0, tile_row(t + 2 * S)), r2_1 = row_of(i2_1, tile_row(t + 2 * S));
      const int i3_0 = idx_at(t + 3 * S, lane), i3_1 = idx_at(t + 3 * S, lane + 32);
      const bool fail = t >= kRing && !mbar_wait(BAR(BAR_IXE + rs), ((t / kRing) - 1) & 1, wl);
      if (__any_sync(0xffffffffu, fail)) break;  // warp-uniform exit
      // rows first (the loaders need only them), then the row scales
      s_row[rs * 64 + lane] = r0_0;
      s_row[rs * 64 + lane + 32] = r0_1;
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_IXF + rs));
      if (kFp8) {
        s_rsc[rs * 64 + lane] = c0_0;
        s_rsc[rs * 64 + lane + 32] = c0_1;
      }
      if (kDsv4) {
        s_dsc[rs * 64 + lane] = d0_0;
        s_dsc[rs * 64 + lane + 32] = d0_1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_IXS + rs));
      r0_0 = r1_0; r0_1 = r1_1;
      c0_0 = c1_0; c0_1 = c1_1;
      d0_0 = d1_0; d0_1 = d1_1;
      r1_0 = r2_0; r1_1 = r2_1;
      i2_0 = i3_0; i2_1 = i3_1;
    }
  } else if (kConv && warp >= kWarpLoad0 + C::kCopyWarps) {
    // ------------------------------------------------------- convert warps
    // fp8 / DeepSeek-V4 caches: turn raw tile t (rows as stored, 576
    // contiguous bytes each) into bf16 operand tile t.  Thread (tok, sub)
    // converts the 16 codes of dims [64 a + 16 sub, +16) of every atom a of
    // row tok (one 16-byte load, two 16-byte stores per atom; a warp's eight
    // rows alternate between the two halves of a 128-byte bank window on the
    // load side and spread over the swizzle on the store side).  Padding
    // rows are written as zeros, whatever the raw slot holds.
    const int ct = threadIdx.x - 32 * (kWarpLoad0 + C::kCopyWarps);  // 0 .. 255
    const int tok = ct >> 2, sub = ct & 3;
    // DeepSeek-V4 pages: atoms 0..6 hold codes (times the group's UE8M0
    // scale), atom 7 the bf16 rope dims, copied as they are
    constexpr int kCvtAtoms = kDsv4 ? kDsv4Nope / 64 : kAtoms;
    constexpr int kRaw = C::kRawStages > 0 ? C::kRawStages : 1;   // (compiled for every kind)
    const uint32_t lo_off = sw128_off(tok, 2 * sub), hi_off = sw128_off(tok, 2 * sub + 1);
    for (int t = 0; t < ntiles; ++t) {
      const int stage = t % kStages, rst = t % kRaw, rs = t % kRing;
      if (__any_sync(0xffffffffu, !mbar_wait(BAR(BAR_IXS + rs), (t / kRing) & 1, wl))) break;
      const bool valid = s_row[rs * 64 + tok] >= 0;
      const uint2 dsc = kDsv4 ? s_dsc[rs * 64 + tok] : make_uint2(0u, 0u);
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_IXE + rs));
      if (__any_sync(0xffffffffu, !mbar_wait(BAR(BAR_RAW + rst), (t / kRaw) & 1, wl))) break;
      if (__any_sync(0xffffffffu, t >= kStages && !mbar_wait(BAR(BAR_KVE + stage), ((t / kStages) - 1) & 1, wl)))
        break;
      // the last operand stage first holds the staged query
      if (__any_sync(0xffffffffu, t == C::kQStage && !mbar_wait(BAR(BAR_QT), 0, wl))) break;
      const uint32_t rrow = sbase + C::kSmemRaw + rst * kRawTileBytes + tok * kRawRowBytes;
      const uint32_t tbase = sbase + kSmemKV + stage * kTileBytes;
      // all loads first (independent), then convert and store
      uint4 v[kCvtAtoms];
#pragma unroll
      for (int a = 0; a < kCvtAtoms; ++a) v[a] = ld_shared_v4(rrow + sub * 16 + a * 64);
#pragma unroll
      for (int a = 0; a < kCvtAtoms; ++a) {
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = make_uint4(0u, 0u, 0u, 0u);
        if (valid) {
          if constexpr (kDsv4) {
            const uint32_t s2 = ue8m0_bf16x2(((a < 4 ? dsc.x : dsc.y) >> (8 * (a & 3))) & 0xFFu);
            e4m3x4_to_bf16x4_scaled(v[a].x, s2, lo.x, lo.y);
            e4m3x4_to_bf16x4_scaled(v[a].y, s2, lo.z, lo.w);
            e4m3x4_to_bf16x4_scaled(v[a].z, s2, hi.x, hi.y);
            e4m3x4_to_bf16x4_scaled(v[a].w, s2, hi.z, hi.w);
          } else {
            e4m3x4_to_bf16x4(v[a].x, lo.x, lo.y);
            e4m3x4_to_bf16x4(v[a].y, lo.z, lo.w);
            e4m3x4_to_bf16x4(v[a].z, hi.x, hi.y);
            e4m3x4_to_bf16x4(v[a].w, hi.z, hi.w);
          }
        }
        st_shared_v4(tbase + a * kAtomBytes + lo_off, lo);
        st_shared_v4(tbase + a * kAtomBytes + hi_off, hi);
      }
      if constexpr (kDsv4) {
        // rope: bf16 bytes [448 + 32 sub, +32) of the slot, chunks 2 sub and
        // 2 sub + 1 of atom 7
        uint4 lo = ld_shared_v4(rrow + kDsv4Nope + 32 * sub);
        uint4 hi = ld_shared_v4(rrow + kDsv4Nope + 32 * sub + 16);
        if (!valid) lo = hi = make_uint4(0u, 0u, 0u, 0u);
        st_shared_v4(tbase + 7 * kAtomBytes + lo_off, lo);
        st_shared_v4(tbase + 7 * kAtomBytes + hi_off, hi);
      }
      // one proxy fence for the tile: generic stores -> tensor-core reads
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(BAR(BAR_KVF + stage));
        mbar_arrive(BAR(BAR_RAWE + rst));
      }
    }
  } else if (warp >= kWarpLoad0) {
    // ------------------------------------------------------- copy warps
    // Each warp instruction covers eight rows, four 16-byte chunks of each
    // (lane = 4 row + chunk): spreading an instruction over many rows keeps
    // more DRAM requests independent, which measured faster on B200 than
    // whole-row instructions.  Copy warp lw owns the 8-row groups
    // g = lw + kCopyWarps i of every tile.  Padding rows read nothing
    // (source size 0).
    constexpr int kGpw = 8 / C::kCopyWarps;          // groups per copy warp
    const int lt = threadIdx.x - 32 * kWarpLoad0;  // 0 .. kCopy-1
    const int lw = lt >> 5;
    const int r8 = lane >> 2, c4 = lane & 3;
    for (int t = 0; t < ntiles; ++t) {
      const int stage = t % kStages, rs = t % kRing;
      if (__any_sync(0xffffffffu, !mbar_wait(BAR(BAR_IXF + rs), (t / kRing) & 1, wl))) break;  // warp-uniform
      // this lane's row in each of the warp's groups, and, for a bulk group,
      // the row of lane l < 8
      int rows[kGpw], brow[kGpw];
#pragma unroll
      for (int gi = 0; gi < kGpw; ++gi) {
        rows[gi] = s_row[rs * 64 + 8 * (lw + C::kCopyWarps * gi) + r8];
        brow[gi] = s_row[rs * 64 + 8 * (lw + C::kCopyWarps * gi) + (lane & 7)];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_IXE + rs));
      if constexpr (kNat) {
        if (__any_sync(0xffffffffu, t >= kStages && !mbar_wait(BAR(BAR_KVE + stage), ((t / kStages) - 1) & 1, wl)))
          break;
        // the last two stages first hold the staged query
        if (__any_sync(0xffffffffu, (t == C::kQStage || t == C::kQStage + 1) && !mbar_wait(BAR(BAR_QT), 0, wl)))
          break;
        // fp8 rows as stored, into the core-matrix layout: chunk c (0..35)
        // of a row to cm_off(row in tile, c).  One instruction per row for
        // its first 512 bytes (lane = chunk), then one for the last 64 bytes
        // of the group's eight rows (lane = 4 row + chunk - 32): per 128-byte
        // line of a gathered row this issues fewer requests than eight rows x
        // 64 bytes per instruction, which measured ~7 % faster on 576-byte
        // rows although each 512-byte instruction meets bank conflicts on
        // the shared-memory side.
        const uint32_t tbase = sbase + kSmemKV + stage * C::kOpBytes;
#pragma unroll
        for (int gi = 0; gi < kGpw; ++gi) {
          const int g = lw + C::kCopyWarps * gi;
#pragma unroll
          for (int rr = 0; rr < 8; ++rr) {
            const int row = __shfl_sync(0xffffffffu, rows[gi], 4 * rr);   // lane 4 rr holds row 8 g + rr
            const uint8_t* src = p.kv + (size_t)(row >= 0 ? row : 0) * kRowBytesFp8;
            cp_async_16(tbase + cm_off(8 * g + rr, lane), src + lane * 16, row >= 0 ? 16u : 0u);
          }
          {
            const int row = rows[gi];                                     // row 8 g + r8
            const uint8_t* src = p.kv + (size_t)(row >= 0 ? row : 0) * kRowBytesFp8;
            cp_async_16(tbase + cm_off(8 * g + r8, 32 + c4), src + (32 + c4) * 16, row >= 0 ? 16u : 0u);
          }
        }
        cp_async_mbar_arrive_noinc(BAR(BAR_KVF + stage));
      } else if constexpr (!kConv) {
        if (__any_sync(0xffffffffu, t >= kStages && !mbar_wait(BAR(BAR_KVE + stage), ((t / kStages) - 1) & 1, wl)))
          break;
        // the last stage first holds the staged query
        if (__any_sync(0xffffffffu, t == C::kQStage && !mbar_wait(BAR(BAR_QT), 0, wl))) break;
        // bf16 rows straight into the swizzled operand tile: chunk c (0..71)
        // of a row is 16-byte chunk c % 8 of atom c / 8.  Two instructions
        // per row for its first 1,024 bytes (lane = chunk), then two for the
        // last 128 bytes of the group's eight rows (lane = 8 row + chunk - 64
        // over four rows each).
        const uint32_t tbase = sbase + kSmemKV + stage * kTileBytes;
        auto copy_chunk = [&](int tok, int row, int c) {
          const uint8_t* src = p.kv + (size_t)(row >= 0 ? row : 0) * kRowBytesBf16;
          cp_async_16(tbase + (c >> 3) * kAtomBytes + sw128_off(tok, c & 7), src + c * 16, row >= 0 ? 16u : 0u);
        };
#pragma unroll
        for (int gi = 0; gi < kGpw; ++gi) {
          const int g = lw + C::kCopyWarps * gi;
#pragma unroll
          for (int rr = 0; rr < 8; ++rr) {
            const int row = __shfl_sync(0xffffffffu, rows[gi], 4 * rr);   // lane 4 rr holds row 8 g + rr
            copy_chunk(8 * g + rr, row, lane);
            copy_chunk(8 * g + rr, row, 32 + lane);
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int rr = 4 * hh + (lane >> 3);
            copy_chunk(8 * g + rr, __shfl_sync(0xffffffffu, rows[gi], 4 * rr), 64 + (lane & 7));
          }
        }
        cp_async_mbar_arrive_noinc(BAR(BAR_KVF + stage));
      } else {
        // raw rows, 576 contiguous bytes each, into raw stage t % 2: groups
        // g < kCpGroups by cp.async, the others one bulk copy per row
        const int rst = t % C::kRawStages;
        if (__any_sync(0xffffffffu, t >= C::kRawStages &&
                                        !mbar_wait(BAR(BAR_RAWE + rst), ((t / C::kRawStages) - 1) & 1, wl)))
          break;
        const uint32_t rbase = sbase + C::kSmemRaw + rst * kRawTileBytes;
        auto row_src = [&](int r) -> const uint8_t* {
          if constexpr (kDsv4) return p.kv + (size_t)(r >> 6) * kDsv4Page + (r & 63) * kDsv4Slot;
          else return p.kv + (size_t)r * kRowBytesFp8;
        };
#pragma unroll
        for (int gi = 0; gi < kGpw; ++gi) {
          const int g = lw + C::kCopyWarps * gi;
          if (g >= C::kCpGroups) {
            // bulk group: lane l < 8 copies row 8 g + l when it is valid
            const bool v = lane < 8 && brow[gi] >= 0;
            const uint32_t nv = __popc(__ballot_sync(0xffffffffu, v));
            if (lane == 0) mbar_arrive_expect_tx(BAR(BAR_RAW + rst), nv * (uint32_t)kRawRowBytes);
            __syncwarp();
            if (v) bulk_load_g2s(rbase + (8 * g + lane) * kRawRowBytes, row_src(brow[gi]), kRawRowBytes, BAR(BAR_RAW + rst));
          } else {
            // one instruction per row for its first 512 bytes (lane =
            // chunk), one for the last 64 bytes of the group's eight rows
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              const int row = __shfl_sync(0xffffffffu, rows[gi], 4 * rr);   // lane 4 rr holds row 8 g + rr
              cp_async_16(rbase + (8 * g + rr) * kRawRowBytes + lane * 16, row_src(row >= 0 ? row : 0) + lane * 16,
                          row >= 0 ? 16u : 0u);
            }
            const int row = rows[gi];                                       // row 8 g + r8
            cp_async_16(rbase + (8 * g + r8) * kRawRowBytes + (32 + c4) * 16, row_src(row >= 0 ? row : 0) + (32 + c4) * 16,
                        row >= 0 ? 16u : 0u);
          }
        }
        cp_async_mbar_arrive_noinc(BAR(BAR_RAW + rst));
      }
    }
    cp_async_wait_all();
  } else if (warp == kWarpS || warp == kWarpPV || warp == C::kWarpS2 || warp == C::kWarpPV2) {
    // ------------------------------------------------------------ MMA issuers
    // Warps that issue tensor-core work, each blocking (in hardware) on one
    // barrier at a time: warp kWarpS computes S(t) once tile t has landed
    // (fp8: its first half, then kWarpS2 the second once the first has
    // completed); warp kWarpPV computes PV(t) once P(t) is written (fp8:
    // dims 0-255, kWarpPV2 dims 256-511).  Each warp runs with warp-uniform
    // state and one elected lane issues; tcgen05.commit tracks the issuing
    // thread's own MMAs.  Operand addresses advance by constants (shared
    // descriptors: byte offset >> 4; tensor memory: columns).
    auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
      return __shfl_sync(0xffffffffu, (int)mbar_wait(bar, parity, wl), 0) != 0;
    };
    bool ok = true;
    if (C::kSplitIss && warp == C::kWarpS2) {
      // the second half of S(t): the query's low part (K steps 18-35),
      // accumulated once the high part has completed
      for (int t = 0; ok && t < ntiles; ++t) {
        const int stage = t % kStages, sb = t % kNumS;
        ok = wait_all(BAR(BAR_SH + sb), (t / kNumS) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + kColS + 64u * (uint32_t)sb;
        const uint64_t bk = cm_desc(sbase + kSmemKV + stage * C::kOpBytes, 128, kCmGroupBytes);
#pragma unroll
        for (int k = kDqk / 32; k < 2 * kDqk / 32; ++k)
          mma8_ts_elect(d, tmem + kColQ + 8u * (uint32_t)k, bk + (uint64_t)((k % 18) * 16), kIdescS8, true);
        commit_elect(BAR(BAR_SF + sb));
      }
    } else if (warp == kWarpS) {
      const uint64_t dk0 = sw128_desc(sbase + kSmemKV, 16, 1024);
      // (stall_test: the cluster barrier, which nothing arrives on without a
      // cluster, stands in for the query: the wait runs out, no MMA is
      // issued, and every other warp's wait runs out in turn)
      ok = wait_all(BAR(p.stall_test ? BAR_CS1 : BAR_QT), 0);
      tc_fence_after();
      int seg = 0;   // rows begun (stream-K)
      for (int t = 0; ok && t < ntiles; ++t) {
        const int stage = t % kStages, sb = t % kNumS;
        if (sk && t > 0 && tile_in_row(t) == 0) {
          // tile t begins the next row: its query replaces the last one in
          // tensor memory (written once the last row's scores were read)
          ++seg;
          ok = wait_all(BAR(BAR_QT), (uint32_t)(seg & 1));
          if (!ok) break;
          tc_fence_after();
        }
        // S(t) reuses the S buffer of S(t-kNumS): its softmax must have read
        // it.  (Nothing else orders S(t) after the PV MMAs before it: issued
        // as soon as its buffer is free, S(t) is done by the time the
        // softmax reaches tile t, which measured faster than holding it
        // behind PV(t-2).)
        if (t >= kNumS) {
          ok = wait_all(BAR(BAR_SE + sb), ((t / kNumS) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
        }
        ok = wait_all(BAR(BAR_KVF + stage), (t / kStages) & 1);
        if (!ok) break;
        const uint32_t d = tmem + kColS + 64u * (uint32_t)sb;
        if constexpr (kNat) {
          // 36 K steps of 32 codes: the query's high part (steps 0-17), then
          // its low part (18-35, issued by kWarpS2), each against K chunks
          // 2 (k mod 18) and +1 (+256 B, +16 in the descriptor); Q columns +8
          // per step
          const uint64_t bk = cm_desc(sbase + kSmemKV + stage * C::kOpBytes, 128, kCmGroupBytes);
          mma8_ts_elect(d, tmem + kColQ, bk, kIdescS8, false);
#pragma unroll
          for (int k = 1; k < (C::kSplitIss ? 1 : 2) * kDqk / 32; ++k)
            mma8_ts_elect(d, tmem + kColQ + 8u * (uint32_t)k, bk + (uint64_t)((k % 18) * 16), kIdescS8, true);
        } else {
          // stage s starts s * kTileBytes later (descriptor address field: bytes >> 4)
          const uint64_t bk = dk0 + (uint64_t)(stage * (kTileBytes >> 4));
          // 36 K steps: Q columns +8 per step (16 bf16); K descriptor: atom
          // +512, 16-element step +2
          mma_ts_set_elect(d, tmem + kColQ, bk, kIdescS);
#pragma unroll
          for (int k = 1; k < kQK / 16; ++k) {
            const uint64_t off = (uint64_t)((k >> 2) * (kAtomBytes >> 4) + (k & 3) * 2);
            mma_ts_acc_elect(d, tmem + kColQ + 8u * (uint32_t)k, bk + off, kIdescS);
          }
        }
        commit_elect(BAR((C::kSplitIss ? BAR_SH : BAR_SF) + sb));
      }
    } else {
      const uint64_t dv0 = sw128_desc(sbase + kSmemKV, kAtomBytes, 1024);
      // (fp8: this warp's half of the output dims)
      const int hf0 = C::kSplitIss && warp == C::kWarpPV2 ? 1 : 0, hf1 = C::kSplitIss ? hf0 + 1 : 2;
      const uint32_t o0 = tmem + (kLaneO << 16);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int stage = t % kStages;
        ok = wait_all(BAR(BAR_PF + stage), (t / kStages) & 1);
        if (!ok) break;
        tc_fence_after();
        const bool fresh = t == 0 || (sk && tile_in_row(t) == 0);   // O starts over (a row's first tile)
        if constexpr (kNat) {
          // O[:, 256 hf + n] += P8[:, 32 kk + k] V[32 (kk mod 2) + k, 256 hf + n]:
          // A = P buffer t mod 4 (codes 0-63: high parts of the 64 tokens,
          // 64-127: low parts; K step +32 B), B = the stage's codes
          // MN-major (8-token groups 4608 B apart, 16-dim chunks 128 B
          // apart; dims 256 hf = chunk 16 hf)
          const uint32_t vb = sbase + kSmemKV + stage * C::kOpBytes;
          const uint64_t dp = sw128_desc(sbase + C::kSmemP + (t & 3) * kAtomBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int hf = hf0; hf < hf1; ++hf) {
              const uint64_t bb = cm_desc(vb + (uint32_t)(((4 * (kk & 1)) * (kRawRowBytes / 16) + 16 * hf) * 128),
                                          kCmGroupBytes, 128);
              mma8_ss_elect(o0 + 256u * (uint32_t)hf, dp + (uint64_t)(2 * kk), bb, kIdescPV8, !fresh || kk > 0);
            }
          }
        } else {
          const uint64_t bv = dv0 + (uint64_t)(stage * (kTileBytes >> 4));
          // P(t) sits in the stage's rope atom
          const uint64_t dp = sw128_desc(sbase + kSmemKV + stage * kTileBytes + kAtomP * kAtomBytes, 16, 1024);
          // O[:, 256 hf + n] += P[:, 16 kk + k] V[16 kk + k, 256 hf + n]:
          // A = P (K step +32 B), B = V MN-major (tokens +2048 B, dims 256
          // = four atoms = +32768 B)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const uint32_t d = o0 + 256u * (uint32_t)hf;
              const uint64_t a = dp + (uint64_t)(2 * kk);
              const uint64_t bb = bv + (uint64_t)(128 * kk + 2048 * hf);
              if (fresh && kk == 0) mma_set_elect(d, a, bb, kIdescPV);
              else mma_acc_elect(d, a, bb, kIdescPV);
            }
          }
        }
        commit_elect(BAR(BAR_KVE + stage));
        commit_elect(BAR(BAR_PVD + (t & 3)));
      }
    }
    // drain: every MMA this warp issued has completed before teardown
    const int fin = warp == kWarpS ? BAR_FIN : warp == kWarpPV ? BAR_FIN2 : warp == C::kWarpS2 ? BAR_FIN3 : BAR_FIN4;
    commit_elect(BAR(fin));
    mbar_wait(BAR(fin), 0);
  } else if (warp < kSmx) {
    // ------------------------------------------------------------ softmax
    // kSmx warps; warp w reaches tensor-memory lane quarter q = w % 4 (heads
    // 16 q .. 16 q + 15).  Thread (w, lane) owns head h = 16 q + lane % 16
    // and, of every tile, the kTok tokens [32 half + kTok u, +kTok) (half =
    // lane / 16, u = w / 4); of O it holds dims [256 half, +256), 32-dim
    // chunks [kOc u, kOc u + kOc).  With two warps per quarter a head's
    // maxima and sums are combined through shared memory at a barrier of
    // the quarter's two warps (named barrier 2 + q), which also ORs their
    // abort flags: both leave the tile loop at the same tile.
    constexpr int kU = kSmx / 4, kTok = 32 / kU, kOc = 8 / kU;
    const int q = warp & 3, u = warp >> 2;
    const int h = 16 * q + (lane & 15);
    const int half = lane >> 4;
    const int tok0 = 32 * half + kTok * u;
    const uint32_t q_lanes = (uint32_t)(32 * q) << 16;            // Q / S rows
    const uint32_t o_lanes = (uint32_t)(32 * q + kLaneO) << 16;   // O rows
    float* s_xch = reinterpret_cast<float*>(smem + C::kAuxXch);   // [2 slots][kU][64]
    int xc = 0;                                                   // exchanges so far
    // v combined over the kU warps of head h (max or sum; v already
    // combined over the thread's two halves), abort flags ORed
    auto pair_reduce = [&](float v, bool is_max, bool& ab) -> float {
      if constexpr (kU == 1) {
        ab = __any_sync(0xffffffffu, ab);
        return v;
      } else {
        float* x = s_xch + (xc & 1) * (2 * 64);
        ++xc;
        if (lane < 16) x[u * 64 + h] = v;
        ab = group_any(ab, 2 + q, 64);
        const float o = x[(1 - u) * 64 + h];
        return is_max ? fmaxf(v, o) : v + o;
      }
    };
    // fp8: 2^-sq, the power of two the head's query was scaled by
    float q_unscale = 1.f;
    bool aborted = false;
    float* s_qsc = reinterpret_cast<float*>(smem + C::kAuxQsc);
    // fp8 (warps u == 0): decode row r's query into tensor memory as e4m3
    // parts: x = q * 2^sq (the head's largest |q| scaled into [128, 256)),
    // high part e4m3(x) at columns [0, 144), low part e4m3(x - high) at
    // [144, 288); this thread's dims [288 half, +288) are columns
    // [72 half, +72) of each.  Read twice (the scale first) from the copy
    // staged in shared memory (the CTA's first row), or else straight from
    // global memory.  Then the scale goes to s_qsc for the quarter's other
    // warp and the warp arrives on BAR_QT.
    auto load_query = [&](int r, bool staged) {
      const uint4* qg = reinterpret_cast<const uint4*>(p.q + ((size_t)r * kH + h) * (kDqk * 2) + half * kDqk);
      const uint32_t qs = sbase + kSmemKV + C::kQStage * C::kOpBytes + (uint32_t)(h * (kDqk * 2) + half * kDqk);
      auto q16 = [&](int k4) -> uint4 { return staged ? ld_shared_v4(qs + 16u * (uint32_t)k4) : __ldg(qg + k4); };
      uint32_t amax = 0;   // largest |q| as bf16 magnitude bits (ordered like the values)
#pragma unroll 4
      for (int k = 0; k < kDqk / 16; ++k) {
        // (staged: lane-rotated order, so that the half-warp's 16 head
        // rows, 1152 bytes apart, meet in different banks)
        const int k4 = staged ? (k + lane) % (kDqk / 16) : k;
        const uint4 v = q16(k4);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) amax = max(amax, max(w4[k] & 0x7FFFu, (w4[k] >> 16) & 0x7FFFu));
      }
      amax = max(amax, (uint32_t)__shfl_xor_sync(0xffffffffu, (int)amax, 16));
      const float qmax = __uint_as_float(amax << 16);
      const int sq = qmax > 0.f ? min(126, max(-126, 7 - ilog2f(qmax))) : 0;   // (subnormal maxima: 126)
      const float qscale = pow2i(sq);
      q_unscale = pow2i(-sq);
#pragma unroll 1
      for (int c = 0; c < kDqk / 64; ++c) {   // 32 dims per step
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint4 v = q16(4 * c + k4);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; k += 2) {
            uint32_t h0, l0, h1, l1;
            split_e4m3x2(__uint_as_float(w4[k] << 16) * qscale, __uint_as_float(w4[k] & 0xFFFF0000u) * qscale,
                         h0, l0);
            split_e4m3x2(__uint_as_float(w4[k + 1] << 16) * qscale,
                         __uint_as_float(w4[k + 1] & 0xFFFF0000u) * qscale, h1, l1);
            hw[2 * k4 + k / 2] = h0 | (h1 << 16);
            lw[2 * k4 + k / 2] = l0 | (l1 << 16);
          }
        }
        tmem_st_16x32bx2_x8<72>(tmem + q_lanes + kColQ + 8u * (uint32_t)c, hw);
        tmem_st_16x32bx2_x8<72>(tmem + q_lanes + kColQ + 144u + 8u * (uint32_t)c, lw);
      }
      tmem_wait_st();
      if (lane < 16) s_qsc[h] = q_unscale;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_QT));
    };
    if constexpr (kNat) {
      if (u == 0) {
        if (!mbar_wait(BAR(BAR_QS), 0)) aborted = true;
        load_query(b0, true);
      } else {
        // the other warp of the quarter takes the head's scale once the
        // query is in place
        if (!mbar_wait(BAR(BAR_QT), 0, wl)) aborted = true;
        q_unscale = s_qsc[h];
      }
    } else if (u == 0) {
      // the query row into tensor memory: dims [kQK/2 half, +kQK/2), read
      // from the copy staged in shared memory (row-major [64][kQK])
      bool okq = mbar_wait(BAR(BAR_QS), 0);
      if (okq) {
        const uint8_t* qrow = smem + kSmemKV + C::kQStage * kTileBytes + h * (kQK * 2) + half * kQK;
#pragma unroll 1
        for (int c = 0; c < kQK / 64; ++c) {
          uint32_t r[16];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint4 v = *reinterpret_cast<const uint4*>(qrow + c * 64 + k4 * 16);
            r[4 * k4] = v.x; r[4 * k4 + 1] = v.y; r[4 * k4 + 2] = v.z; r[4 * k4 + 3] = v.w;
          }
          tmem_st_16x32bx2_x16<kQK / 4>(tmem + q_lanes + kColQ + 16u * (uint32_t)c, r);  // second half at +kQK/4
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_QT));
    }
    // l_run: sum of the probabilities as fp32 (gives lse); l_pv: the same sum
    // of the bf16-rounded probabilities the PV MMA used (normalises out, so
    // the output weights sum to one exactly).
    float m_run = -INFINITY, l_run = 0.f, l_pv = 0.f;
    // fp8: O and its normaliser are kept times sig2 (0 until the first
    // nonzero probability), the power of two of the e4m3 P parts
    float sig2 = 0.f;
    float fsc = p.scale_log2 * q_unscale;
    // stream-K: the row being computed, its first tile here, rows begun
    int srow = b0, sfirst = 0, seg = 0;
    // both warps of the quarter (the named barrier of the pair)
    auto pair_sync = [&]() {
      if constexpr (kU == 2) named_bar_sync(2 + q, 64);
      else __syncwarp();
    };
    // Stream-K: row r's result from this CTA's tiles [t0, t1).  A row that
    // lies wholly in this CTA is written out straight from tensor memory.
    // Otherwise each of the CTAs that hold part of it (a piece) counts
    // itself in at the row's counter (one per lane quarter, so the quarters
    // never wait for one another); the last piece to arrive merges: every
    // other piece has left its result, normalised, and its lse in its slot
    // (slot 2 j for the first row of CTA j, 2 j + 1 for its last), and the
    // last piece adds them to its own, weighted by 2^(lse - max), as the
    // log-sum-exp combine does.  No CTA waits for another.  The counter
    // holds (epoch << 8) | arrivals; a tag other than this launch's reads as
    // zero arrivals, and the last piece sets it back to 0, so the workspace
    // needs no initialisation.
    auto finish_row = [&](int r, int t0, int t1) {
      if (!aborted) {
        // PV(t1-2) then PV(t1-1): each wait is at most one phase ahead
        if (t1 - t0 >= 2 && !mbar_wait(BAR(BAR_PVD + ((t1 - 2) & 3)), ((t1 - 2) >> 2) & 1, wl)) aborted = true;
        if (!mbar_wait(BAR(BAR_PVD + ((t1 - 1) & 3)), ((t1 - 1) >> 2) & 1, wl)) aborted = true;
        tc_fence_after();
      }
      float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      l_tot = pair_reduce(l_tot, false, aborted);
      if (aborted) return;
      const float l_nrm = l_tot * sig2;
      const float inv_l = l_tot > 0.f && l_nrm > 0.f ? 1.f / l_nrm : 0.f;
      const float lse2 = l_tot > 0.f ? m_run + log2f(l_tot) : -INFINITY;   // log2 units
      const long long W = (long long)p.batch * nt;
      const long long G = gridDim.x;
      auto owner = [&](long long g) -> int { return (int)(((g + 1) * G - 1) / W); };   // CTA of global tile g
      const int j0 = owner((long long)r * nt), j1 = owner((long long)(r + 1) * nt - 1);
      __nv_bfloat16* orow = p.out + ((size_t)r * kH + h) * kDv;
      if (j0 == j1) {
#pragma unroll 1
        for (int c = kOc * u; c < kOc * (u + 1); ++c) {
          float o[32];
          tmem_ld_16x32bx2_x32_h256(tmem + o_lanes + 32u * (uint32_t)c, o);
          tmem_wait_ld();
          uint4* dst = reinterpret_cast<uint4*>(orow + half * 256 + c * 32);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            dst[k4] = make_uint4(pack_bf16x2(o[8 * k4] * inv_l, o[8 * k4 + 1] * inv_l),
                                 pack_bf16x2(o[8 * k4 + 2] * inv_l, o[8 * k4 + 3] * inv_l),
                                 pack_bf16x2(o[8 * k4 + 4] * inv_l, o[8 * k4 + 5] * inv_l),
                                 pack_bf16x2(o[8 * k4 + 6] * inv_l, o[8 * k4 + 7] * inv_l));
        }
        if (u == 0 && half == 0) p.lse[(size_t)r * kH + h] = lse2 * 0.6931471805599453f;
        return;
      }
      const unsigned npc = (unsigned)(j1 - j0 + 1);
      const unsigned long long ep = p.epoch;
      unsigned long long* ctr = p.row_ctr + (size_t)r * 4 + q;
      int* s_flag = reinterpret_cast<int*>(smem + C::kAuxFlag);
      // 1. has every other piece arrived already?  Then this one merges
      //    without leaving its own result.
      if (u == 0 && lane == 0) {
        const unsigned long long v = ld_relaxed_gpu_u64(ctr);
        const unsigned c = (v >> 8) == ep ? (unsigned)(v & 255u) : 0u;
        const int lastp = c + 1 == npc;
        if (lastp) {
          __threadfence();
          atomicExch(ctr, 0ull);
        }
        s_flag[q] = lastp;
      }
      pair_sync();
      bool last = s_flag[q] != 0;
      if (!last) {
        // 2. this piece's result (normalised) and lse to its slot, then
        //    count it in
        const int slot = 2 * (int)blockIdx.x + (r == b0 ? 0 : 1);
        float* so = p.part_o + ((size_t)slot * kH + h) * kDv;
#pragma unroll 1
        for (int c = kOc * u; c < kOc * (u + 1); ++c) {
          float o[32];
          tmem_ld_16x32bx2_x32_h256(tmem + o_lanes + 32u * (uint32_t)c, o);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(so + half * 256 + c * 32);
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4)
            dst[k4] = make_float4(__fmul_rn(o[4 * k4], inv_l), __fmul_rn(o[4 * k4 + 1], inv_l),
                                  __fmul_rn(o[4 * k4 + 2], inv_l), __fmul_rn(o[4 * k4 + 3], inv_l));
        }
        if (u == 0 && half == 0) p.part_lse[(size_t)slot * kH + h] = lse2;
        __threadfence();
        pair_sync();
        if (u == 0 && lane == 0) {
          unsigned long long v = ld_relaxed_gpu_u64(ctr);
          int lastp = -1;
          // (each failed exchange is another piece's arrival: at most npc - 1)
          for (int it = 0; it < 64; ++it) {
            const unsigned c = (v >> 8) == ep ? (unsigned)(v & 255u) : 0u;
            const unsigned long long nv = c + 1 == npc ? 0ull : ((ep << 8) | (unsigned long long)(c + 1));
            const unsigned long long pv = atomicCAS(ctr, v, nv);
            if (pv == v) {
              lastp = c + 1 == npc ? 1 : 0;
              break;
            }
            v = pv;
          }
          if (lastp < 0) atomicOr(&g_error_word, 1u);
          if (lastp == 1) __threadfence();
          s_flag[q] = lastp == 1;
        }
        pair_sync();
        last = s_flag[q] != 0;
      }
      if (!last) return;
      // 3. merge, in the order of the pieces (CTA j0 first) whichever
      //    merges, so the result does not depend on the order of arrival:
      //    the pieces' lse and weights, then per 32-dim chunk their
      //    normalised results (from L2; this piece's from tensor memory,
      //    normalised as it would have been stored) weighted and summed
      //    with one rounding per product and per sum
      const int self = (int)blockIdx.x;
      float lk[kMaxPieces];
      const float* po[kMaxPieces];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < kMaxPieces; ++k) {
        const int j = j0 + k;
        lk[k] = -INFINITY;
        po[k] = nullptr;
        if (j == self) {
          lk[k] = lse2;
        } else if (j <= j1) {
          const long long first_g = (long long)j * W / G;   // CTA j's first tile
          const int sl = 2 * j + (first_g / nt == r ? 0 : 1);
          lk[k] = __ldcg(p.part_lse + (size_t)sl * kH + h);
          po[k] = p.part_o + ((size_t)sl * kH + h) * kDv + half * 256;
        }
        mx = fmaxf(mx, lk[k]);
      }
      float wk[kMaxPieces], wsum = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxPieces; ++k) {
        wk[k] = lk[k] == -INFINITY ? 0.f : ex2(lk[k] - mx);
        wsum = __fadd_rn(wsum, wk[k]);
      }
      const float inv_w = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll 1
      for (int c = kOc * u; c < kOc * (u + 1); ++c) {
        float o[32];
        tmem_ld_16x32bx2_x32_h256(tmem + o_lanes + 32u * (uint32_t)c, o);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(orow + half * 256 + c * 32);
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {   // 8 dims at a time
          float acc[8];
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) acc[e2] = 0.f;
#pragma unroll
          for (int k = 0; k < kMaxPieces; ++k) {
            const float f = __fmul_rn(wk[k], inv_w);
            if (j0 + k == self) {
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2)
                acc[e2] = __fadd_rn(acc[e2], __fmul_rn(f, __fmul_rn(o[8 * g8 + e2], inv_l)));
            } else if (po[k] != nullptr) {
              const float4* src = reinterpret_cast<const float4*>(po[k] + c * 32 + 8 * g8);
              const float4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
              const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2) acc[e2] = __fadd_rn(acc[e2], __fmul_rn(f, v[e2]));
            }
          }
          dst[g8] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                               pack_bf16x2(acc[6], acc[7]));
        }
      }
      if (u == 0 && half == 0)
        p.lse[(size_t)r * kH + h] = wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
    };
    for (int i = 0; i < ntiles; ++i) {
      if (sk && i > 0 && tile_in_row(i) == 0) {
        // Tile i begins the next row.  The quarter's two warps agree to go
        // on; the next row's query goes to tensor memory first (the last
        // row's scores have all been read, and the next row's first scores
        // are then computed during this epilogue), then the last row's
        // result is written and the running state starts over.
        if constexpr (kU == 2) aborted = group_any(aborted, 2 + q, 64);
        else aborted = __any_sync(0xffffffffu, aborted);
        if (aborted) break;
        ++seg;
        if (u == 0) load_query(srow + 1, false);
        finish_row(srow, sfirst, i);
        if (u != 0) {
          if (!mbar_wait(BAR(BAR_QT), (uint32_t)(seg & 1), wl)) aborted = true;
          q_unscale = s_qsc[h];
        }
        m_run = -INFINITY;
        l_run = 0.f;
        l_pv = 0.f;
        sig2 = 0.f;
        fsc = p.scale_log2 * q_unscale;
        ++srow;
        sfirst = i;
      }
      const int sb = i % kNumS, rs = i % kRing;
      if (!mbar_wait(BAR(BAR_SF + sb), (i / kNumS) & 1, wl) || !mbar_wait(BAR(BAR_IXS + rs), (i / kRing) & 1, wl))
        aborted = true;
      aborted = __any_sync(0xffffffffu, aborted);
      float s[kTok];
      if (!aborted) {
        tc_fence_after();
        if constexpr (kTok == 32) tmem_ld_16x32bx2_x32(tmem + q_lanes + kColS + 64u * (uint32_t)sb, s);
        else tmem_ld_16x32bx2_x16(tmem + q_lanes + kColS + 64u * (uint32_t)sb + (uint32_t)(kTok * u), s);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < kTok; ++j) s[j] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_SE + sb));

      int rows[kTok];
      float rsc[kTok];
#pragma unroll
      for (int j = 0; j < kTok; j += 4) {
        const int4 r4 = *reinterpret_cast<const int4*>(s_row + rs * 64 + tok0 + j);
        rows[j] = r4.x; rows[j + 1] = r4.y; rows[j + 2] = r4.z; rows[j + 3] = r4.w;
        if (kFp8) {
          const float4 c4 = *reinterpret_cast<const float4*>(s_rsc + rs * 64 + tok0 + j);
          rsc[j] = c4.x; rsc[j + 1] = c4.y; rsc[j + 2] = c4.z; rsc[j + 3] = c4.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_IXE + rs));
      // logits in log2 units (padding: -inf) and this thread's maximum
      float tm[kTok / 2];
#pragma unroll
      for (int j = 0; j < kTok; ++j) {
        const float f = kFp8 ? fsc * rsc[j] : p.scale_log2;
        s[j] = rows[j] >= 0 ? s[j] * f : -INFINITY;
      }
#pragma unroll
      for (int j = 0; j < kTok / 2; ++j) tm[j] = fmaxf(s[2 * j], s[2 * j + 1]);
#pragma unroll
      for (int w2 = kTok / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int j = 0; j < w2; ++j) tm[j] = fmaxf(tm[j], tm[j + w2]);
      // Probabilities against the running maximum, as long as no thread's
      // logits pass it by more than the lazy threshold and (fp8) no thread's
      // P' = p rsc leaves the range of the current power of two sig2.  One
      // barrier of the quarter's warps tells whether any of their threads
      // needs an update (or gave up a wait); only then are the heads' exact
      // maxima exchanged and the probabilities recomputed.
      float pr[kTok];
      float lsum = 0.f, lsum_pv = 0.f;
      uint32_t pk[kTok / 2];
      auto probabilities = [&](float m_ref) -> float {   // returns this thread's largest |P'|
        float pmx = 0.f;
        lsum = 0.f;
        lsum_pv = 0.f;
#pragma unroll
        for (int j = 0; j < kTok; j += 2) {
          const float p0 = s[j] == -INFINITY ? 0.f : ex2(s[j] - m_ref);
          const float p1 = s[j + 1] == -INFINITY ? 0.f : ex2(s[j + 1] - m_ref);
          lsum += p0 + p1;
          if constexpr (kNat) {
            pr[j] = p0 * rsc[j];
            pr[j + 1] = p1 * rsc[j + 1];
            pmx = fmaxf(pmx, fmaxf(fabsf(pr[j]), fabsf(pr[j + 1])));
          } else {
            const uint32_t w = pack_bf16x2(p0, p1);
            pk[j / 2] = w;
            lsum_pv += __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
          }
        }
        return pmx;
      };
      // (every finite logit needs an update while m_run = -inf; the values
      // computed against m_run are then discarded)
      bool upd = tm[0] > m_run + kRescaleThresh;
      float pmax = probabilities(upd ? tm[0] : m_run);
      if constexpr (kNat) upd = upd || (pmax > 0.f && (sig2 == 0.f || pmax * sig2 >= 448.f));
      float m_use = m_run, alpha = 1.f, r = 1.f;
      bool need = false;
      bool slow;
      if constexpr (kU == 1) slow = __any_sync(0xffffffffu, upd || aborted);
      else slow = group_any(upd || aborted, 2 + q, 64);
      if (slow) {
        // the head's maximum over its 2 kU threads, then P against it
        float tmax = fmaxf(tm[0], __shfl_xor_sync(0xffffffffu, tm[0], 16));
        tmax = pair_reduce(tmax, true, aborted);
        if (aborted) break;
        const float m_new = fmaxf(m_run, tmax);
        need = m_new > m_run + kRescaleThresh;
        m_use = need ? m_new : m_run;
        alpha = need ? ex2(m_run - m_use) : 1.f;
        pmax = probabilities(m_use);
        if constexpr (kNat) {
          // P' goes to the MMA as e4m3 parts of P' sig2.  sig2 is set at the
          // first tile with mass (its largest |P'| into [8, 16): values down
          // to 2^-10 of it keep the parts' full 8 bits, and later tiles may
          // grow 28-fold before anything changes) and lowered by a power of
          // two r when a later tile's largest value would pass the e4m3
          // maximum 448 (again into [8, 16)); O then takes the same factor.
          pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 16));
          pmax = pair_reduce(pmax, true, aborted);
          if (pmax > 0.f) {
            if (sig2 == 0.f) {
              sig2 = pow2i(min(126, max(-126, 3 - ilog2f(pmax))));
            } else {
              const float tp = pmax * sig2;
              if (tp >= 448.f) {
                r = pow2i(max(-126, 3 - ilog2f(tp)));
                sig2 *= r;
              }
            }
          }
        }
      }
      // Rescale this head's O row (this thread's chunks) by alpha r.  Only
      // then must PV(i-1) have completed.  PVD[(i-1) mod 4] is at most one
      // phase behind: PV(i-5) has completed (bf16 operands: tile i was
      // loaded after PV(i-3) released its stage; fp8: this warp waited for
      // PV(i-5) before writing P(i-1)), and PV(i+3) needs P(i+3).
      const bool resc_m = need && i >= 1 && m_run > -INFINITY;
      const bool resc = resc_m || r != 1.f;
      if (__any_sync(0xffffffffu, resc)) {
        if (!mbar_wait(BAR(BAR_PVD + ((i - 1) & 3)), ((i - 1) >> 2) & 1, wl)) aborted = true;
        aborted = __any_sync(0xffffffffu, aborted);
        if (!aborted) {
          tc_fence_after();
          const float f = (resc_m ? alpha : 1.f) * r;
#pragma unroll 1
          for (int c = kOc * u; c < kOc * (u + 1); ++c) {
            float o[32];
            const uint32_t ta = tmem + o_lanes + 32u * (uint32_t)c;
            tmem_ld_16x32bx2_x32_h256(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= f;
            tmem_st_16x32bx2_x32_h256(ta, o);
          }
          tmem_wait_st();
        }
      }
      l_run = l_run * alpha + lsum;
      l_pv = l_pv * alpha + lsum_pv;
      m_run = m_use;
      uint32_t prow;
      if constexpr (kNat) {
        // high and low e4m3 parts, four tokens per word
        uint32_t hw[kTok / 4], lw[kTok / 4];
#pragma unroll
        for (int j = 0; j < kTok; j += 4) {
          uint32_t h0, l0, h1, l1;
          split_e4m3x2_h(pr[j] * sig2, pr[j + 1] * sig2, h0, l0);
          split_e4m3x2_h(pr[j + 2] * sig2, pr[j + 3] * sig2, h1, l1);
          hw[j / 4] = h0 | (h1 << 16);
          lw[j / 4] = l0 | (l1 << 16);
        }
        // P buffer i mod 4 is free once PV(i-4) has completed (which also
        // keeps the PVD waits of tile i+1 at most one phase ahead)
        if (i >= 4 && !mbar_wait(BAR(BAR_PVD + (i & 3)), ((i - 4) >> 2) & 1, wl)) aborted = true;
        aborted = __any_sync(0xffffffffu, aborted);
        if (aborted) continue;   // (the next exchange, or the epilogue's, stops every softmax warp)
        // row h: codes [tok0, +kTok) high parts (16-token chunks tok0 / 16
        // on), codes [64 + tok0, +kTok) low parts
        prow = sbase + C::kSmemP + (uint32_t)((i & 3) * kAtomBytes);
#pragma unroll
        for (int k = 0; k < kTok / 16; ++k) {
          st_shared_v4(prow + sw128_off(h, tok0 / 16 + k), make_uint4(hw[4 * k], hw[4 * k + 1], hw[4 * k + 2], hw[4 * k + 3]));
          st_shared_v4(prow + sw128_off(h, 4 + tok0 / 16 + k),
                       make_uint4(lw[4 * k], lw[4 * k + 1], lw[4 * k + 2], lw[4 * k + 3]));
        }
      } else {
        if (aborted) continue;
        // P(t) [64 heads][64 tokens] bf16 in the stage's rope atom: row h,
        // 8-token chunks tok0 / 8 on
        prow = sbase + kSmemKV + (i % kStages) * kTileBytes + kAtomP * kAtomBytes;
#pragma unroll
        for (int k = 0; k < kTok / 8; ++k)
          st_shared_v4(prow + sw128_off(h, tok0 / 8 + k), make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(BAR_PF + i % kStages));
    }
    // ---------------------------------------------------------- epilogue
    // this CTA's tiles are done: the next kernel of the stream may start
    // on idle SMs (it waits for this grid's completion before reading)
    if (threadIdx.x == 0) grid_dep_launch();
    if (sk) {
      if (ntiles > 0) finish_row(srow, sfirst, ntiles);
    } else {
      if (!aborted && ntiles > 0) {
        // PV(n-2) then PV(n-1): each wait is at most one phase ahead
        if (ntiles >= 2 && !mbar_wait(BAR(BAR_PVD + ((ntiles - 2) & 3)), ((ntiles - 2) >> 2) & 1, wl)) aborted = true;
        if (!mbar_wait(BAR(BAR_PVD + ((ntiles - 1) & 3)), ((ntiles - 1) >> 2) & 1, wl)) aborted = true;
        tc_fence_after();
      }
      // the head's totals over its kU warps (and the common abort decision)
      float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      l_tot = pair_reduce(l_tot, false, aborted);
      // the normaliser of O (bf16 operands: the rounded-P sum; fp8: the
      // probability sum times sig2) and the split's weight in a merge (the
      // rounded-P sum; fp8: the probability sum)
      float l_w = l_tot;
      if constexpr (!kNat) {
        l_w = l_pv + __shfl_xor_sync(0xffffffffu, l_pv, 16);
        l_w = pair_reduce(l_w, false, aborted);
      }
      const float l_nrm = kNat ? l_tot * sig2 : l_w;
      if (p.cluster) {
        // in-cluster merge (after the warp roles): this split's per-head
        // statistics (max, merge weight, fp32 sum) go to the workspace
        merge_failed = aborted;
        if (!aborted && u == 0 && half == 0) {
          float* wss = p.part_lse + (size_t)b * p.nsplit * 64 * kStatFloats;
          *reinterpret_cast<float4*>(wss + ((size_t)split * 64 + h) * kStatFloats) = make_float4(m_run, l_w, l_tot, 0.f);
          // for the merge writers: 1 / (normaliser of O) of head h
          reinterpret_cast<float*>(smem + C::kAuxRow)[h] = l_nrm > 0.f ? 1.f / l_nrm : 0.f;
        }
      } else if (!aborted) {
        const bool any = l_tot > 0.f;
        const float inv_l = any && l_nrm > 0.f ? 1.f / l_nrm : 0.f;
        const float lse_h = any ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
        const bool direct = p.nsplit == 1;
        const size_t part = (size_t)b * p.nsplit + split;
        // Stage the head rows in shared memory (the idle operand stages) with
        // a 16-byte pad per row, which makes the 16-byte stores of a warp
        // conflict-free, then write each row with one bulk copy.
        const uint32_t row_bytes = direct ? kDv * 2 : kDv * 4;
        const uint32_t stride = row_bytes + 16;
        uint8_t* srow = smem + kSmemKV + (size_t)h * stride;
  #pragma unroll 1
        for (int c = kOc * u; c < kOc * (u + 1); ++c) {
          float o[32];
          if (ntiles > 0) {
            tmem_ld_16x32bx2_x32_h256(tmem + o_lanes + 32u * (uint32_t)c, o);
            tmem_wait_ld();
          } else {
  #pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0.f;
          }
          const int d0 = half * 256 + c * 32;   // this thread's 32 dims
          if (direct) {
            uint4* dst = reinterpret_cast<uint4*>(srow + d0 * 2);
  #pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              dst[k4] = make_uint4(pack_bf16x2(o[8 * k4] * inv_l, o[8 * k4 + 1] * inv_l),
                                   pack_bf16x2(o[8 * k4 + 2] * inv_l, o[8 * k4 + 3] * inv_l),
                                   pack_bf16x2(o[8 * k4 + 4] * inv_l, o[8 * k4 + 5] * inv_l),
                                   pack_bf16x2(o[8 * k4 + 6] * inv_l, o[8 * k4 + 7] * inv_l));
          } else {
            float4* dst = reinterpret_cast<float4*>(srow + d0 * 4);
  #pragma unroll
            for (int k4 = 0; k4 < 8; ++k4)
              dst[k4] = make_float4(o[4 * k4] * inv_l, o[4 * k4 + 1] * inv_l, o[4 * k4 + 2] * inv_l,
                                    o[4 * k4 + 3] * inv_l);
          }
        }
        fence_proxy_async_smem();
        // the row's other chunks come from the other warp of the quarter
        if constexpr (kU == 2) named_bar_sync(2 + q, 64);
        else __syncwarp();
        if (u == 0 && half == 0) {
          uint8_t* gdst = direct ? reinterpret_cast<uint8_t*>(p.out + ((size_t)b * kH + h) * kDv)
                                 : reinterpret_cast<uint8_t*>(p.part_o + (part * kH + h) * kDv);
          bulk_store_s2g(gdst, smem_u32(srow), row_bytes);
          bulk_commit();
          if (direct) p.lse[(size_t)b * kH + h] = lse_h;
          else p.part_lse[part * kH + h] = lse_h;
          bulk_wait_all();
        }
      }
    }
    tc_fence_before();
  }

  if (p.cluster && warp < 8) {
    // ------------------------------------- split merge inside the cluster
    // The nsplit CTAs of this sequence form a cluster (rank = split); the
    // exchange goes through the workspace (L2), one launch in all, and
    // warps 0-7 (the softmax warps and, their roles done, warps 4-7, which
    // reach the same tensor-memory lanes: warp w and w + 4 share quarter w)
    // share the work.
    // 1. Each CTA stores its O, unnormalised, straight from tensor memory in
    //    "register image" order ([quarter][chunk][vector][lane], so each
    //    warp store covers 512 contiguous bytes); warps 0-3 take chunks
    //    0-3, warps 4-7 chunks 4-7.  The softmax warps stored the per-head
    //    (m, l, l_pv) already.
    // 2. One cluster-wide barrier: remote mbarrier arrivals (release),
    //    bounded waits (acquire).  Every CTA arrives and waits even after an
    //    error, so no remote arrival targets a CTA that has exited.
    // 3. CTA r owns output columns [r cn, (r+1) cn), cn = 512 / nsplit.
    //    Thread (head hh, part 0-3) reads its cn / 4 columns of every split
    //    (16 lanes x 16 contiguous bytes per load), weights split s by
    //    2^(m_s - M), divides by the equally weighted sum of the rounded-P
    //    sums (the normalisation of one CTA over all tiles) and writes bf16;
    //    rank 0 writes lse.
    const int n = p.nsplit;
    const int q = warp & 3;                                  // tensor-memory lane quarter
    const int upper = warp >> 2;                             // 0: softmax warp, 1: helper warp
    constexpr size_t kSplitU = (size_t)kH * kDv / 8;         // 16-byte units (8 fp16) per split
    uint4* wso = reinterpret_cast<uint4*>(p.part_o) + (size_t)b * n * kSplitU;     // [src][q][c][u][lane]
    float* wss = p.part_lse + (size_t)b * n * 64 * kStatFloats;  // [src][64][8]: m, l_pv, l, -, part scales
    bool failed = merge_failed;
    if (upper) {
      // every PV has completed (the PV issuers' drain barriers: one phase)
      failed = !mbar_wait(BAR(BAR_FIN2), 0) || (C::kSplitIss && !mbar_wait(BAR(BAR_FIN4), 0));
      tc_fence_after();
    }
    const bool bad = group_any(failed, 1, 256);
    if (!bad) {
      // This split's result for the thread's head, normalised by its own
      // rounded-P sum (a convex combination of value rows), times a power of
      // two that puts the largest magnitude of the thread's 128 dims (part
      // 2 half + upper of the row) in [2^14, 2^15), rounded to fp16: any
      // finite value fits, with 11 significant bits (error <= 2^-12 of the
      // part's largest value).  The inverse scale goes to the statistics.
      const float sc = reinterpret_cast<const float*>(smem + C::kAuxRow)[16 * q + (lane & 15)];
      uint4* mine = wso + (size_t)split * kSplitU + (size_t)q * (8 * 4 * 32) + lane;
      const uint32_t olanes = (uint32_t)(32 * q + kLaneO) << 16;
      float o[2][32];
      const int c0 = 4 * upper;
      float mx = 0.f;
      if (ntiles > 0) {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          tmem_ld_16x32bx2_x32_h256(tmem + olanes + 32u * (uint32_t)(c0 + cc), o[0]);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) mx = fmaxf(mx, fabsf(o[0][k]));
        }
      }
      mx *= sc;
      int ex = mx > 0.f ? (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127 : 0;   // mx in [2^ex, 2^(ex+1))
      ex = max(-100, min(ex, 127));
      const float scw = sc * __uint_as_float((uint32_t)(127 + 14 - ex) << 23);
      wss[((size_t)split * 64 + 16 * q + (lane & 15)) * kStatFloats + 4 + 2 * (lane >> 4) + upper] =
          __uint_as_float((uint32_t)(127 - 14 + ex) << 23);
      if (ntiles > 0) {
        tmem_ld_16x32bx2_x32_h256(tmem + olanes + 32u * (uint32_t)c0, o[0]);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) { o[0][k] = 0.f; o[1][k] = 0.f; }
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = c0 + cc;
        if (ntiles > 0 && cc + 1 < 4) tmem_ld_16x32bx2_x32_h256(tmem + olanes + 32u * (uint32_t)(c + 1), o[(cc + 1) & 1]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float* x = &o[cc & 1][8 * u];
          mine[(c * 4 + u) * 32] = make_uint4(pack_f16x2(x[0] * scw, x[1] * scw), pack_f16x2(x[2] * scw, x[3] * scw),
                                              pack_f16x2(x[4] * scw, x[5] * scw), pack_f16x2(x[6] * scw, x[7] * scw));
        }
        if (ntiles > 0 && cc + 1 < 4) tmem_wait_ld();
      }
    }
    named_bar_sync(1, 256);
    // lane r of warp 0 arrives on CTA r's barrier: the n remote arrivals go
    // out together (one after another they cost a round trip each)
    // (each arrival is a cluster-scope release: after the CTA barrier it
    // covers every merging thread's stores)
    if (warp == 0) {
      if (lane < n) mbar_arrive_cluster(mapa_shared(BAR(BAR_CS1), (uint32_t)lane));
      __syncwarp();
    }
    const bool ok = mbar_wait_cluster(BAR(BAR_CS1), 0);
    if (!group_any(bad || !ok, 1, 256)) {
      const int hh = 16 * q + (lane & 15);
      const int part = (lane >> 4) + 2 * upper;
      const int cn = kDv / n;                 // columns this CTA reduces
      const int col0 = split * cn + part * (cn / 4);
      __nv_bfloat16* orow = p.out + ((size_t)b * kH + hh) * kDv + col0;
      switch (n) {
        case 2: merge_tail<2>(wss, wso, q, lane, hh, col0, orow); break;
        case 4: merge_tail<4>(wss, wso, q, lane, hh, col0, orow); break;
        case 8: merge_tail<8>(wss, wso, q, lane, hh, col0, orow); break;
        default: merge_tail<16>(wss, wso, q, lane, hh, col0, orow); break;
      }
    }
    tc_fence_before();
  } else if (p.cluster && split == 0 && warp >= 8 && warp < 10) {
    // lse of the merged result, head 32 (warp - 8) + lane, from every
    // split's (m, l) once all have stored them: two index warps of rank 0,
    // idle by now and outside the merging warps 0-7, alongside the column
    // merge
    const int hh = 32 * (warp - 8) + lane;
    const float* wss = p.part_lse + (size_t)b * p.nsplit * 64 * kStatFloats;
    if (mbar_wait_cluster(BAR(BAR_CS1), 0)) {
      float mv[16], lr[16];
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) {
        mv[s2] = -INFINITY;
        lr[s2] = 0.f;
        if (s2 < p.nsplit) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(wss + ((size_t)s2 * 64 + hh) * kStatFloats));
          mv[s2] = v.x; lr[s2] = v.z;
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) M = fmaxf(M, mv[s2]);
      float Lr = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) Lr += mv[s2] > -INFINITY ? ex2(mv[s2] - M) * lr[s2] : 0.f;
      p.lse[(size_t)b * kH + hh] = Lr > 0.f ? (M + log2f(Lr)) * 0.6931471805599453f : -INFINITY;
    }
  }

  __syncthreads();
  if (warp == kWarpS) {
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
  grid_dep_wait();       // the split kernel's partials are complete
  grid_dep_launch();
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

// Query tokens per sequence (0 means one) and decode rows (sequences x tokens).
static int tokens_of(const smla_shape* s) { return s->tokens_per_seq > 1 ? s->tokens_per_seq : 1; }
static int rows_of(const smla_shape* s) { return s->batch * tokens_of(s); }

static smla_status validate_shape(const smla_shape* s) {
  if (!s) return SMLA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535 || s->topk < 1 || s->topk > (1 << 24)) return SMLA_ERR_INVALID_ARG;
  if (s->tokens_per_seq < 0 || s->tokens_per_seq > 16 || (long long)s->batch * tokens_of(s) > 65535)
    return SMLA_ERR_INVALID_ARG;
  if (s->num_kv_rows < 1 || s->num_kv_rows > 0x7FFFFFFFLL) return SMLA_ERR_INVALID_ARG;
  if (s->nsplit < 0 && s->nsplit != SMLA_NSPLIT_STREAMK) return SMLA_ERR_INVALID_ARG;
  if (s->kv_dtype != SMLA_KV_BF16 && s->kv_dtype != SMLA_KV_FP8_E4M3_ROWSCALE && s->kv_dtype != SMLA_KV_DSV4_PAGED)
    return SMLA_ERR_UNSUPPORTED;
  const int want_qk = s->kv_dtype == SMLA_KV_DSV4_PAGED ? 512 : kDqk;
  if (s->num_heads != kH || s->d_qk != want_qk || s->d_v != kDv) return SMLA_ERR_UNSUPPORTED;
  if (s->page_size != 0 && s->page_size != 64) return SMLA_ERR_UNSUPPORTED;
  // DeepSeek-V4 pages hold 64 token slots: paged only, whole pages
  if (s->kv_dtype == SMLA_KV_DSV4_PAGED && (s->page_size != 64 || s->num_kv_rows % 64 != 0))
    return SMLA_ERR_UNSUPPORTED;
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

static int plan_nsplit_raw(const smla_shape* s, int num_sms) {
  const int tiles = (s->topk + kTile - 1) / kTile;
  int n;
  if (s->nsplit > 0) {      // (SMLA_NSPLIT_STREAMK without a stream-K plan: automatic)
    n = s->nsplit;
  } else {
    n = num_sms > 0 ? num_sms / rows_of(s) : 1;
  }
  if (n < 1) n = 1;
  if (n > tiles) n = tiles;
  return n;
}

// The split plan: n CTAs per sequence, each over a contiguous run of tiles.
// cluster: the n CTAs form a thread-block cluster and merge inside the
// split kernel (no combine kernel); possible when n is a power of two no
// larger than 16 that the device can launch as a cluster.  An explicit
// nsplit is kept as given (merged in the kernel whenever it can launch as a
// cluster); an automatic plan takes the largest such n that fits in one
// wave (falling back to one split).
//
// Stream-K (asked for with nsplit = SMLA_NSPLIT_STREAMK): fp8 rows with
// lists of at least 16 tiles, more rows than half the SMs but not a multiple
// of them, are shared out over one CTA per SM: the rows' tiles are laid end
// to end and each CTA takes an equal run (so a row falls to at most three
// CTAs), merged inside the kernel by the CTA that finishes its part of the
// row last.  Other shapes asking for it get the automatic plan.
struct Plan {
  int n;
  bool cluster;
  bool streamk;
};
static bool streamk_fits(const smla_shape* s, int num_sms) {
  if (s->kv_dtype != SMLA_KV_FP8_E4M3_ROWSCALE || s->nsplit != SMLA_NSPLIT_STREAMK || num_sms < 2) return false;
  const long long rows = rows_of(s), nt = (s->topk + kTile - 1) / kTile;
  return nt >= 16 && 2 * rows > num_sms && rows % num_sms != 0 && rows * nt < (1ll << 31);
}
static Plan make_plan(const smla_shape* s, int num_sms, const int active[5], bool allow_streamk = true) {
  Plan pl{plan_nsplit_raw(s, num_sms), false, false};
  if (pl.n < 2) {
    pl.streamk = allow_streamk && streamk_fits(s, num_sms);
    return pl;
  }
  if (s->nsplit > 0) {
    if ((pl.n & (pl.n - 1)) == 0 && pl.n <= 16) pl.cluster = active[31 - __builtin_clz(pl.n)] >= 1;
    return pl;
  }
  // The largest power-of-two split (<= the raw count) whose B clusters are
  // all resident at once; on B200 this measured within a few percent of the
  // best split count for every batch and list length tried.
  for (int lg = 4; lg >= 1; --lg) {
    const int c = 1 << lg;
    if (c <= pl.n && active[lg] >= rows_of(s)) return Plan{c, true, false};
  }
  return Plan{1, false, false};
}

static size_t partial_bytes(int batch, int nsplit) {
  const size_t o = (size_t)batch * nsplit * kH * kDv * 4;
  const size_t l = (size_t)batch * nsplit * kH * 4;
  return ((o + l + 255) / 256) * 256;
}

// Workspace of an in-cluster merge: every split's scaled, normalised result
// (rows * nsplit * 64 * 512 fp16) and its per-head statistics (rows *
// nsplit * 64 * kStatFloats fp32).
static size_t cluster_bytes(int batch, int nsplit) {
  const size_t o = (size_t)batch * nsplit * kH * kDv * 2;
  const size_t st = (size_t)batch * nsplit * kH * kStatFloats * 4;
  return ((o + st + 255) / 256) * 256;
}
static size_t workspace_bytes_for(int batch, int nsplit, bool cluster) {
  if (nsplit < 2) return 0;
  return cluster ? cluster_bytes(batch, nsplit) : partial_bytes(batch, nsplit);
}
// Workspace of a stream-K plan over a grid of g CTAs: two result slots per
// CTA (its first and last row, when another CTA shares them) as fp32
// [2 g, 64, 512], their lse [2 g, 64], then the row counters [rows, 4] u64.
static size_t streamk_o_bytes(int g) { return (((size_t)2 * g * kH * kDv * 4) + 255) / 256 * 256; }
static size_t streamk_lse_bytes(int g) { return (((size_t)2 * g * kH * 4) + 255) / 256 * 256; }
static size_t streamk_bytes(int rows, int g) {
  return streamk_o_bytes(g) + streamk_lse_bytes(g) + (((size_t)rows * 4 * 8) + 255) / 256 * 256;
}
static size_t plan_workspace_bytes(const smla_shape* s, const Plan& pl, int num_sms) {
  return pl.streamk ? streamk_bytes(rows_of(s), num_sms) : workspace_bytes_for(rows_of(s), pl.n, pl.cluster);
}
// A tag per launch for the stream-K row counters (never 0, below 2^56).
static unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{0};
  unsigned long long e = 0;
  while (e == 0) e = (counter.fetch_add(1) + 1) & ((1ull << 56) - 1);
  return e;
}

// The shared-memory opt-in is set once per device (an idempotent call, so a
// race between threads is harmless); later calls, including calls made
// while a stream is being captured into a CUDA graph, skip it.
template <int kKind, bool kSK = false>
static cudaError_t ensure_smem_attr() {
  static volatile int done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(smla_split_kernel<kKind, kSK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg<kKind>::kSmemBytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
  return e;
}

// How many clusters of c split CTAs (c = 2, 4, 8, 16) the device holds at
// once for this kernel (1 CTA per SM: a cluster needs c SMs of one GPC).
// Queried once per device; 0 = that size cannot launch.
struct ClusterCaps {
  int active[5];  // index log2(c); active[0] unused
};
template <int kKind>
static const ClusterCaps& cluster_caps() {
  static ClusterCaps cache[64];
  static volatile int done[64] = {0};
  static ClusterCaps none = {{0, 0, 0, 0, 0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return none;
  if (done[dev]) return cache[dev];
  ClusterCaps caps = {{0, 0, 0, 0, 0}};
  if (ensure_smem_attr<kKind>() == cudaSuccess &&
      cudaFuncSetAttribute(smla_split_kernel<kKind, false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess) {
    for (int lg = 1; lg <= 4; ++lg) {
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 1u << lg;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1u << lg, 1, 1);
      cfg.blockDim = dim3(Cfg<kKind>::kThreads, 1, 1);
      cfg.dynamicSmemBytes = Cfg<kKind>::kSmemBytes;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int k = 0;
      if (cudaOccupancyMaxActiveClusters(&k, smla_split_kernel<kKind, false>, &cfg) == cudaSuccess) caps.active[lg] = k;
    }
  }
  cudaGetLastError();  // a refused query leaves no sticky error
  cache[dev] = caps;
  done[dev] = 1;
  return cache[dev];
}
static const ClusterCaps& caps_for(const smla_shape* s) {
  if (s->kv_dtype == SMLA_KV_FP8_E4M3_ROWSCALE) return cluster_caps<kKindFp8>();
  if (s->kv_dtype == SMLA_KV_DSV4_PAGED) return cluster_caps<kKindDsv4>();
  return cluster_caps<kKindBf16>();
}

template <int kKind>
static cudaError_t launch_split(const SplitParams& prm, int grid_x, cudaStream_t stream) {
  auto kern = smla_split_kernel<kKind, false>;
  cudaError_t e = ensure_smem_attr<kKind>();
  if (e != cudaSuccess) return e;
  if constexpr (kKind == kKindFp8) {
    if (prm.streamk) {
      kern = smla_split_kernel<kKind, true>;
      e = ensure_smem_attr<kKind, true>();
      if (e != cudaSuccess) return e;
    }
  }
  // programmatic dependent launch (the kernel waits for its prerequisites
  // itself), and for an in-cluster merge the cluster of nsplit CTAs
  cudaLaunchAttribute at[2];
  int na = 0;
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (prm.cluster) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = prm.nsplit;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = prm.streamk ? dim3(grid_x, 1) : dim3(prm.nsplit, prm.batch);
  cfg.blockDim = dim3(Cfg<kKind>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg<kKind>::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

static smla_status run_split(const smla_shape* shape, const void* q, const void* kv_cache,
                             const float* kv_row_scale, const int32_t* page_table, const int32_t* indices,
                             float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                             int32_t* nsplit_out, cudaStream_t stream, int* nsplit_used, bool allow_fused,
                             bool* cluster_used, long long wait_limit = kWaitLimitCycles, int stall_test = 0) {
  smla_status st = validate_shape(shape);
  if (st != SMLA_OK) return st;
  if (!q || !kv_cache || !indices || !out || !lse) return SMLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16) || !aligned(indices, 4) || !aligned(lse, 4))
    return SMLA_ERR_INVALID_ARG;
  const bool fp8 = shape->kv_dtype == SMLA_KV_FP8_E4M3_ROWSCALE;
  if (fp8 && (!kv_row_scale || !aligned(kv_row_scale, 4))) return SMLA_ERR_INVALID_ARG;
  if (shape->kv_dtype == SMLA_KV_DSV4_PAGED && kv_row_scale) return SMLA_ERR_INVALID_ARG;
  if (shape->page_size && (!page_table || !aligned(page_table, 4))) return SMLA_ERR_INVALID_ARG;
  if (!(scale == scale) || isinf(scale)) return SMLA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return SMLA_ERR_CUDA;
  // (allow_fused: the in-kernel merges, in a cluster or stream-K, may be used)
  const Plan pl = make_plan(shape, sms, caps_for(shape).active, allow_fused);
  const int n = pl.n;
  const bool cluster = allow_fused && pl.cluster;
  if (n > 1 || pl.streamk) {
    if (!workspace || !aligned(workspace, 256)) return SMLA_ERR_WORKSPACE;
    const size_t need = pl.streamk ? streamk_bytes(rows_of(shape), sms) : workspace_bytes_for(rows_of(shape), n, cluster);
    if (workspace_bytes < need) return SMLA_ERR_WORKSPACE;
  }
  SplitParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.q = static_cast<const uint8_t*>(q);
  prm.kv = static_cast<const uint8_t*>(kv_cache);
  prm.kv_row_scale = kv_row_scale;
  prm.page_table = page_table;
  prm.num_kv_rows = (int)shape->num_kv_rows;
  prm.indices = indices;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.cluster = cluster ? 1 : 0;
  prm.part_o = static_cast<float*>(workspace);
  prm.part_lse = n > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                  (size_t)rows_of(shape) * n * kH * kDv * (cluster ? 2 : 4))
                       : nullptr;
  prm.batch = rows_of(shape);
  prm.tok_per_seq = tokens_of(shape);
  prm.topk = shape->topk;
  prm.nsplit = n;
  prm.ntiles_total = (shape->topk + kTile - 1) / kTile;
  prm.page_size = shape->page_size;
  prm.pages_per_seq = shape->pages_per_seq;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
  prm.wait_limit = wait_limit;
  prm.stall_test = stall_test;
  if (pl.streamk) {
    prm.streamk = 1;
    prm.epoch = next_epoch();
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    prm.part_o = reinterpret_cast<float*>(ws);
    prm.part_lse = reinterpret_cast<float*>(ws + streamk_o_bytes(sms));
    prm.row_ctr = reinterpret_cast<unsigned long long*>(ws + streamk_o_bytes(sms) + streamk_lse_bytes(sms));
  }
  const cudaError_t e = fp8 ? launch_split<kKindFp8>(prm, sms, stream)
                            : (shape->kv_dtype == SMLA_KV_DSV4_PAGED ? launch_split<kKindDsv4>(prm, sms, stream)
                                                                    : launch_split<kKindBf16>(prm, sms, stream));
  if (e != cudaSuccess) return SMLA_ERR_CUDA;
  if (nsplit_out) *nsplit_out = n;
  if (nsplit_used) *nsplit_used = n;
  if (cluster_used) *cluster_used = cluster;
  return SMLA_OK;
}

static smla_status run_combine(int batch, int nsplit, const float* part_o, const float* part_lse, void* out,
                               float* lse, cudaStream_t stream) {
  dim3 grid(kH, batch);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128, 1, 1);
  cfg.stream = stream;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, smla_combine_kernel, part_o, part_lse,
                                           static_cast<__nv_bfloat16*>(out), lse, nsplit);
  return e == cudaSuccess ? SMLA_OK : SMLA_ERR_CUDA;
}

// Device address of g_static_scratch on the current device, looked up once
// per device (with that device current) and kept.
static smla_status static_scratch_address(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SMLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SMLA_ERR_CUDA;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return SMLA_OK;
}

// Device staging of sparse_mla_decode_host: q, indices, page table, out,
// lse and the decode workspace, each region 256-byte aligned.
struct HostStaging {
  size_t q, q_bytes, idx, idx_bytes, pt, pt_bytes, out, out_bytes, lse, lse_bytes, ws, ws_bytes, total;
};
static size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
static HostStaging host_staging(const smla_shape* s, size_t ws_bytes) {
  HostStaging h;
  size_t off = 0;
  h.q_bytes = (size_t)rows_of(s) * kH * s->d_qk * 2;
  h.idx_bytes = (size_t)rows_of(s) * s->topk * 4;
  h.pt_bytes = s->page_size ? (size_t)s->batch * s->pages_per_seq * 4 : 0;
  h.out_bytes = (size_t)rows_of(s) * kH * kDv * 2;
  h.lse_bytes = (size_t)rows_of(s) * kH * 4;
  h.ws_bytes = ws_bytes;
  h.q = off;   off += round256(h.q_bytes);
  h.idx = off; off += round256(h.idx_bytes);
  h.pt = off;  off += round256(h.pt_bytes);
  h.out = off; off += round256(h.out_bytes);
  h.lse = off; off += round256(h.lse_bytes);
  h.ws = off;  off += round256(h.ws_bytes);
  h.total = off;
  return h;
}

}  // namespace smla

// the indexer step (scores and top-k selection), sharing the helpers above
#include "indexer.cuh"

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
    case SMLA_ERR_DEVICE_INDEX: return "SMLA_ERR_DEVICE_INDEX";
    case SMLA_ERR_DEVICE_LAYOUT: return "SMLA_ERR_DEVICE_LAYOUT";
  }
  return "SMLA_ERR_UNKNOWN";
}

int32_t sparse_mla_plan_nsplit(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return 0;
  return smla::make_plan(shape, smla::device_sm_count(), smla::caps_for(shape).active).n;
}

size_t sparse_mla_workspace_size(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return 0;
  const int sms = smla::device_sm_count();
  const smla::Plan pl = smla::make_plan(shape, sms, smla::caps_for(shape).active);
  return smla::plan_workspace_bytes(shape, pl, sms);
}

int32_t sparse_mla_plan_merge(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return -1;
  const smla::Plan pl = smla::make_plan(shape, smla::device_sm_count(), smla::caps_for(shape).active);
  if (pl.streamk) return 3;
  return pl.n < 2 ? 0 : (pl.cluster ? 1 : 2);
}

smla_status sparse_mla_decode_split(const smla_shape* shape, const void* q, const void* kv_cache,
                                    const float* kv_row_scale, const int32_t* page_table,
                                    const int32_t* indices, float scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, int32_t* nsplit_out,
                                    void* stream) {
  return smla::run_split(shape, q, kv_cache, kv_row_scale, page_table, indices, scale, out, lse, workspace,
                         workspace_bytes, nsplit_out, static_cast<cudaStream_t>(stream), nullptr, false, nullptr);
}

smla_status sparse_mla_decode(const smla_shape* shape, const void* q, const void* kv_cache,
                              const float* kv_row_scale, const int32_t* page_table, const int32_t* indices,
                              float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream) {
  int n = 0;
  bool cluster = false;
  const smla_status st = smla::run_split(shape, q, kv_cache, kv_row_scale, page_table, indices, scale, out, lse,
                                         workspace, workspace_bytes, nullptr, static_cast<cudaStream_t>(stream),
                                         &n, true, &cluster);
  if (st != SMLA_OK || n == 1 || cluster) return st;
  const float* po = static_cast<const float*>(workspace);
  const float* pl = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) +
                                                   (size_t)smla::rows_of(shape) * n * smla::kH * smla::kDv * 4);
  return smla::run_combine(smla::rows_of(shape), n, po, pl, out, lse, static_cast<cudaStream_t>(stream));
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

smla_status sparse_mla_decode_static_scratch(const smla_shape* shape, const void* q, const void* kv_cache,
                                             const float* kv_row_scale, const int32_t* page_table,
                                             const int32_t* indices, float scale, void* out, float* lse,
                                             void* stream) {
  smla_status st = smla::validate_shape(shape);
  if (st != SMLA_OK) return st;
  // split count and scratch need.  No CUDA call when the caller fixes an
  // nsplit whose results fit neither way: the in-cluster merge (possible
  // for a power of two <= 16, whether the device can launch it or not) needs
  // the smaller workspace, the separate combine the larger.
  if (shape->nsplit > 0) {
    const int n0 = smla::plan_nsplit_raw(shape, 0);
    const bool pow2 = n0 > 1 && (n0 & (n0 - 1)) == 0 && n0 <= 16;
    if (n0 > 1 && smla::workspace_bytes_for(smla::rows_of(shape), n0, pow2) > SMLA_STATIC_SCRATCH_BYTES)
      return SMLA_ERR_WORKSPACE;
  }
  const int sms = smla::device_sm_count();
  if (sms <= 0) return SMLA_ERR_CUDA;
  // (the split plan: a stream-K plan's workspace is larger than the scratch)
  const smla::Plan pl = smla::make_plan(shape, sms, smla::caps_for(shape).active, false);
  const int n = pl.n;
  const size_t need = smla::workspace_bytes_for(smla::rows_of(shape), n, pl.cluster);
  if (need > SMLA_STATIC_SCRATCH_BYTES) return SMLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    st = smla::static_scratch_address(&scratch);
    if (st != SMLA_OK) return st;
  }
  // the planned count, fixed, so the launch uses exactly the checked size
  smla_shape fixed = *shape;
  fixed.nsplit = n;
  return sparse_mla_decode(&fixed, q, kv_cache, kv_row_scale, page_table, indices, scale, out, lse, scratch,
                           need, stream);
}

size_t sparse_mla_host_staging_size(const smla_shape* shape) {
  if (smla::validate_shape(shape) != SMLA_OK) return 0;
  return smla::host_staging(shape, sparse_mla_workspace_size(shape)).total;
}

smla_status sparse_mla_decode_host(const smla_shape* shape, const void* q_host, const void* kv_cache,
                                   const float* kv_row_scale, const int32_t* page_table_host,
                                   const int32_t* indices_host, float scale, void* out_host, float* lse_host,
                                   void* staging, size_t staging_bytes, void* stream) {
  smla_status st = smla::validate_shape(shape);
  if (st != SMLA_OK) return st;
  // every argument check before the first copy is enqueued
  if (!q_host || !kv_cache || !indices_host || !out_host || !lse_host) return SMLA_ERR_INVALID_ARG;
  if (!smla::aligned(kv_cache, 16)) return SMLA_ERR_INVALID_ARG;
  if ((shape->page_size != 0) != (page_table_host != nullptr)) return SMLA_ERR_INVALID_ARG;
  const bool fp8 = shape->kv_dtype == SMLA_KV_FP8_E4M3_ROWSCALE;
  if (fp8 != (kv_row_scale != nullptr)) return SMLA_ERR_INVALID_ARG;
  if (fp8 && !smla::aligned(kv_row_scale, 4)) return SMLA_ERR_INVALID_ARG;
  if (!(scale == scale) || isinf(scale)) return SMLA_ERR_INVALID_ARG;
  if (!staging || !smla::aligned(staging, 256)) return SMLA_ERR_WORKSPACE;
  const size_t ws = sparse_mla_workspace_size(shape);
  const smla::HostStaging h = smla::host_staging(shape, ws);
  if (staging_bytes < h.total) return SMLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(staging);
  // one copy per tensor (host to device), the step, then the results back
  if (cudaMemcpyAsync(base + h.q, q_host, h.q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(base + h.idx, indices_host, h.idx_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      (h.pt_bytes && cudaMemcpyAsync(base + h.pt, page_table_host, h.pt_bytes, cudaMemcpyHostToDevice, s) !=
                         cudaSuccess))
    return SMLA_ERR_CUDA;
  st = sparse_mla_decode(shape, base + h.q, kv_cache, kv_row_scale,
                         h.pt_bytes ? reinterpret_cast<const int32_t*>(base + h.pt) : nullptr,
                         reinterpret_cast<const int32_t*>(base + h.idx), scale, base + h.out,
                         reinterpret_cast<float*>(base + h.lse), ws ? base + h.ws : nullptr, ws, stream);
  if (st != SMLA_OK) return st;
  if (cudaMemcpyAsync(out_host, base + h.out, h.out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(lse_host, base + h.lse, h.lse_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SMLA_ERR_CUDA;
  return SMLA_OK;
}

smla_status sparse_mla_decode_stalled(const smla_shape* shape, const void* q, const void* kv_cache,
                                      const int32_t* indices, float scale, void* out, float* lse,
                                      int64_t wait_limit_cycles, void* stream) {
  smla_status st = smla::validate_shape(shape);
  if (st != SMLA_OK) return st;
  if (shape->kv_dtype != SMLA_KV_BF16 || shape->page_size != 0) return SMLA_ERR_UNSUPPORTED;
  if (wait_limit_cycles < 1000 || wait_limit_cycles > smla::kWaitLimitCycles) return SMLA_ERR_INVALID_ARG;
  // one CTA per sequence: no partials, no workspace, no cluster
  smla_shape one = *shape;
  one.nsplit = 1;
  return smla::run_split(&one, q, kv_cache, nullptr, nullptr, indices, scale, out, lse, nullptr, 0, nullptr,
                         static_cast<cudaStream_t>(stream), nullptr, false, nullptr, (long long)wait_limit_cycles, 1);
}

smla_status sparse_mla_get_device_error(uint32_t* code) {
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, smla::g_error_word, sizeof(w)) != cudaSuccess) return SMLA_ERR_CUDA;
  const unsigned int zero = 0;
  if (w != 0 && cudaMemcpyToSymbol(smla::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SMLA_ERR_CUDA;
  if (code) *code = w;
  if (w & 1u) return SMLA_ERR_DEVICE_TIMEOUT;
  if (w & 2u) return SMLA_ERR_DEVICE_LAYOUT;
  if (w & 4u) return SMLA_ERR_DEVICE_INDEX;
  return SMLA_OK;
}

}  // extern "C"
