// Indexer step: the scores that choose the decode's top-k index list, and
// the top-k selection itself.  Included by sparse_mla.cu after the decode
// kernels (same translation unit: the PTX helpers and the device error word
// are shared).
//
// Pages (titles): "The Pivot Point: When a 6.3x Kernel Speedup Reveals the
// Next Bottleneck" -- "The Context: A Campaign in Full Swing" (the indexer's
// batched matrix product belongs on bf16 tensor cores), "Input Knowledge
// Required" (the indexer picks the top ~512 cache positions per decode step;
// the decode attends to those only); "The Moment of Truth: Benchmarking a
// Custom MMA Kernel for DeepSeek-V4-Flash on Blackwell" -- "Broader Context"
// (score only the real context length, not the maximum context).
//
// Scores (the published form of DeepSeek's sparse-attention indexer; the
// pages name only the batched product and the top-k):
//   I[b, s] = sum_h w[b, h] * max(0, q[b, h, :] . k[row(b, s), :]),  s < ctx[b]
// with 64 heads of 128 bf16 dims and the keys in a 64-token paged cache.
// Selection: the min(topk, ctx[b]) largest scores, ties to the lower
// position, positions ascending, -1 after.

namespace smla {

constexpr int kIxH = 64;                         // indexer heads
constexpr int kIxD = 128;                        // dims per head (bf16)
constexpr int kIxTile = 128;                     // positions per CTA (MMA M)
constexpr int kIxThreads = 128;
constexpr int kIxQBytes = kIxH * kIxD * 2;       // 16,384
constexpr int kIxKBytes = kIxTile * kIxD * 2;    // 32,768
constexpr int kIxAtomQ = kIxH * 128;             // one 64-dim half of Q: 64 rows x 128 B
constexpr int kIxAtomK = kIxTile * 128;          // one 64-dim half of K: 128 rows x 128 B
constexpr int kIxSmemQ = 0;
constexpr int kIxSmemK = kIxSmemQ + kIxQBytes;
constexpr int kIxSmemW = kIxSmemK + kIxKBytes;   // w [64] fp32
constexpr int kIxSmemBar = kIxSmemW + kIxH * 4;  // mbarrier: the MMA (8 B)
constexpr int kIxSmemBarK = kIxSmemBar + 8;      // mbarrier: the key copies (8 B)
constexpr int kIxSmemTmem = kIxSmemBarK + 8;     // tensor-memory base address (4 B)
constexpr int kIxSmemBytes = kIxSmemTmem + 8;    // 49,432: four CTAs per SM
constexpr uint32_t kIxTmemCols = 64;             // D: 128 lanes (positions) x 64 columns (heads)
constexpr uint32_t kIdescIx = make_idesc(128, 64, false, false);
static_assert(kIxSmemK % 1024 == 0 && kIxAtomQ % 1024 == 0 && kIxAtomK % 1024 == 0,
              "128B-swizzled operands need 1024-byte aligned atoms");

constexpr int kTkThreads = 1024;                 // top-k: one CTA per sequence

// the C ABI struct as the Python binding lays it out
static_assert(sizeof(smla_indexer_shape) == 40 && offsetof(smla_indexer_shape, num_key_rows) == 32,
              "smla_indexer_shape layout");

struct alignas(64) IndexerParams {
  // the key cache as a 2-D tensor map: [num_rows][128] bf16, box 64 dims x
  // 64 rows, 128-byte swizzle (one half of a page lands as one operand atom)
  CUtensorMap kmap;
  const uint8_t* q;            // [B, 64, 128] bf16
  const float* w;              // [B, 64]
  const uint8_t* k;            // [num_rows, 128] bf16
  const int32_t* page_table;   // [B, pages_per_seq]
  const int32_t* ctx_len;      // [B]
  float* scores;               // [B, max_ctx]
  int max_ctx, pages_per_seq;
  long long num_rows;
};

// 32 lanes x 32 columns: thread t reads columns [c, c+32) of lane base+t.
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

// One CTA per (tile of 128 positions, sequence).  The tile's keys (two
// pages, each 64 contiguous rows of 256 B) come by tensor copies (four, one
// per page and 64-dim half, 128-byte swizzle applied by the copy engine),
// the sequence's query by 16-byte cp.async, both K-major; one elected
// thread issues
// D[128 x 64] = K . Q^T (eight K steps of 16) into tensor memory; then
// thread t of warp w takes position 32 w + t: its 64 head dot products,
// ReLU, weighted by w and summed in fp32, head by head.  Positions past the
// context (and tiles wholly past it) get -inf.
__global__ void __launch_bounds__(kIxThreads) smla_indexer_score_kernel(const __grid_constant__ IndexerParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tile = blockIdx.x, b = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  grid_dep_wait();   // the query, weights and lengths may come from the previous kernel
  int ctx = __ldg(p.ctx_len + b);
  if (ctx < 0 || ctx > p.max_ctx) {
    if (t == 0) atomicOr(&g_error_word, 4u);
    ctx = ctx < 0 ? 0 : p.max_ctx;
  }
  const int s0 = tile * kIxTile;
  float* srow = p.scores + (size_t)b * p.max_ctx;
  if (s0 >= ctx || (sbase & 1023u)) {
    if ((sbase & 1023u) && t == 0) atomicOr(&g_error_word, 2u);
    if (s0 + t < p.max_ctx) srow[s0 + t] = -INFINITY;
    return;
  }
  const uint32_t bar = sbase + kIxSmemBar, bark = sbase + kIxSmemBarK;
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_init(bark, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(sbase + kIxSmemTmem, kIxTmemCols);
    tmem_relinquish();
  }
  // the query: 1,024 chunks of 16 B; chunk c is dims [8 (c % 16), +8) of
  // head c / 16, and goes to half (c % 16) / 8 of the swizzled operand
  const uint8_t* qb = p.q + (size_t)b * kIxQBytes;
#pragma unroll
  for (int u = 0; u < kIxQBytes / 16 / kIxThreads; ++u) {
    const int c = u * kIxThreads + t;
    const int row = c >> 4, j = c & 15;
    cp_async_16(sbase + kIxSmemQ + (j >> 3) * kIxAtomQ + sw128_off(row, j & 7), qb + (size_t)c * 16, 16u);
  }
  // the keys: positions s0 .. s0 + 127 lie in pages s0 / 64 and s0 / 64 + 1
  // of the sequence (the host keeps max_ctx <= 64 pages_per_seq).  A page
  // at or past the context, or outside the cache, is zero-filled instead
  // (its positions score -inf, or 0 when within the context: read as absent).
  long long rbase[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    rbase[h] = -1;
    if (s0 + 64 * h < ctx) {
      const long long e = __ldg(p.page_table + (size_t)b * p.pages_per_seq + (s0 >> 6) + h);
      if (e >= 0 && e * 64 + 64 <= p.num_rows) rbase[h] = e * 64;
      else if (t == 0) atomicOr(&g_error_word, 4u);   // page outside the cache: read as absent
    }
  }
  if (t == 0) {
    const uint32_t nk = (rbase[0] >= 0 ? 2u : 0u) + (rbase[1] >= 0 ? 2u : 0u);
    mbar_arrive_expect_tx(bark, nk * 64u * 128u);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rbase[h] < 0) continue;
#pragma unroll
      for (int half = 0; half < 2; ++half)
        tma_load_2d(sbase + kIxSmemK + half * kIxAtomK + h * 64 * 128, &p.kmap, 64 * half, (int)rbase[h], bark);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (rbase[h] >= 0) continue;
#pragma unroll
    for (int u = 0; u < 2 * 64 * 128 / 16 / kIxThreads; ++u) {
      const int c = u * kIxThreads + t;                 // 16-byte unit of the page's two halves
      st_shared_v4(sbase + kIxSmemK + (c >> 9) * kIxAtomK + h * 64 * 128 + (c & 511) * 16, make_uint4(0u, 0u, 0u, 0u));
    }
  }
  float* ws = reinterpret_cast<float*>(smem + kIxSmemW);
  if (t < kIxH) ws[t] = __ldg(p.w + (size_t)b * kIxH + t);
  cp_async_wait_all();
  fence_proxy_async_smem();   // generic-proxy writes -> tensor-core reads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kIxSmemTmem);
  // the key copies have landed (every thread waits: the copy engine's writes
  // are then visible to the MMA issued below)
  const bool keys_ok = mbar_wait(bark, 0);
  if (warp == 0 && keys_ok) {
    const uint64_t da = sw128_desc(sbase + kIxSmemK, 16, 1024);
    const uint64_t db = sw128_desc(sbase + kIxSmemQ, 16, 1024);
#pragma unroll
    for (int ks = 0; ks < kIxD / 16; ++ks) {
      // 16 dims per step: +32 B inside a 128-byte row, then the next half
      const uint64_t ao = (uint64_t)((ks >> 2) * (kIxAtomK >> 4) + (ks & 3) * 2);
      const uint64_t bo = (uint64_t)((ks >> 2) * (kIxAtomQ >> 4) + (ks & 3) * 2);
      if (ks == 0) mma_set_elect(tmem, da + ao, db + bo, kIdescIx);
      else mma_acc_elect(tmem, da + ao, db + bo, kIdescIx);
    }
    commit_elect(bar);
  }
  const bool ok = keys_ok && mbar_wait(bar, 0);
  tc_fence_after();
  float acc = 0.f;
  if (ok) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float x[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + 32u * (uint32_t)half, x);
      tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 32; ++h) acc = fmaf(ws[32 * half + h], fmaxf(x[h], 0.f), acc);
    }
  }
  const int s = s0 + 32 * warp + lane;
  // + 0.0f turns a -0 sum into +0, so equal scores compare equal as keys
  if (s < p.max_ctx) srow[s] = (ok && s < ctx) ? acc + 0.0f : -INFINITY;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kIxTmemCols);
  if (t == 0) grid_dep_launch();
}

// float -> uint32 whose unsigned order is the float order (+0 and -0 alike)
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix count of `flag` over the block's 1,024 threads (in thread
// order); *total receives the block's count.  sums: 65 ints of shared memory.
__device__ __forceinline__ int block_prefix_count(bool flag, int* sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) sums[warp] = __popc(m);
  __syncthreads();
  if (warp == 0) {
    const int v = sums[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    sums[32 + lane] = incl - v;
    if (lane == 31) sums[64] = incl;
  }
  __syncthreads();
  const int r = sums[32 + warp] + __popc(m & ((1u << lane) - 1u));
  *total = sums[64];
  __syncthreads();   // sums is reused by the next call
  return r;
}

// Warp 0 (t < 32) of a top-k CTA: given the histogram of one 8-bit digit
// over the keys still in play, the digit that holds the need-th largest key
// (*s_digit) and how many keys equal to the selection are still to take
// among those with that digit (*s_need).  Lane l holds digits 255 - 8 l ..
// 248 - 8 l, highest first.
__device__ __forceinline__ void radix_pick(const uint32_t* hist, int need, uint32_t* s_digit, int* s_need) {
  const int t = threadIdx.x;
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    c[k] = hist[255 - 8 * t - k];
    sum += c[k];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (t >= o) incl += v;
  }
  const uint32_t before = incl - sum;   // keys in higher digits
  if (before < (uint32_t)need && (uint32_t)need <= incl) {
    uint32_t acc = before;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (acc + c[k] >= (uint32_t)need) {
        *s_digit = 255u - 8u * (uint32_t)t - (uint32_t)k;
        *s_need = need - (int)acc;
        break;
      }
      acc += c[k];
    }
  }
}

// The same over 2,048 bins (an 11-bit digit), by all 1,024 threads of the
// block: thread t holds bins 2047 - 2 t and 2046 - 2 t (highest first); a
// warp scan and a scan of the 32 warp totals give each thread the number of
// keys in higher bins.  Also sets *s_cnt, the keys that carry the chosen
// digit.  wsum: 32 ints of shared memory.  Ends with the block synchronised.
__device__ __forceinline__ void radix_pick2048(const uint32_t* hist, int need, int* wsum, uint32_t* s_digit,
                                               int* s_need, int* s_cnt) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c0 = (int)hist[2047 - 2 * t], c1 = (int)hist[2046 - 2 * t];
  const int sum = c0 + c1;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = wsum[lane];
    int wi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    __syncwarp();
    wsum[lane] = wi - v;   // keys in the bins of lower-numbered warps
  }
  __syncthreads();
  const int before = wsum[warp] + incl - sum;
  if (before < need && need <= before + sum) {
    if (before + c0 >= need) {
      *s_digit = 2047u - 2u * (uint32_t)t;
      *s_need = need - before;
      *s_cnt = c0;
    } else {
      *s_digit = 2046u - 2u * (uint32_t)t;
      *s_need = need - before - c0;
      *s_cnt = c1;
    }
  }
  __syncthreads();
}

// Warp 0: exclusive prefix sums, in place, of the 256 counts v[0 .. 255];
// returns the total to every lane of warp 0.
__device__ __forceinline__ int prefix256(int* v) {
  const int lane = threadIdx.x & 31;
  int x[8], sum = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[k] = v[8 * lane + k];
    sum += x[k];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - sum;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[8 * lane + k] = run;
    run += x[k];
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// One CTA per sequence.  Radix select of the topk-th largest key, digit by
// digit from the top (histograms in shared memory); then the positions
// above that key, and the lowest positions equal to it until topk are
// taken, written in ascending order.  Contexts up to 8,192 keep their keys
// in registers (position k * 1024 + thread, k < 8): one read of the scores,
// three digits of 11/11/10 bits, and an ordered compaction that ranks by
// (k, warp, lane) through 256-entry prefix sums of per-warp ballot counts.
// Longer contexts re-read the scores for each of four 8-bit digits (one
// atomic per run of equal digits in a warp) and compact 1,024 positions at
// a time.
constexpr int kTkPer = 8;   // keys per thread in registers

__global__ void __launch_bounds__(kTkThreads, 1) smla_topk_kernel(const float* __restrict__ scores,
                                                               const int32_t* __restrict__ ctx_len, int max_ctx,
                                                               int topk, int32_t* __restrict__ out) {
  __shared__ uint32_t hist[2048];
  __shared__ int cnt[256];            // [k][warp] counts, then their prefix sums
  __shared__ int sums[65];
  __shared__ uint32_t s_digit;
  __shared__ int s_need, s_cnt;
  grid_dep_wait();   // the scores come from the previous kernel
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int n = __ldg(ctx_len + b);
  if (n < 0 || n > max_ctx) {
    if (t == 0) atomicOr(&g_error_word, 4u);
    n = n < 0 ? 0 : max_ctx;
  }
  const float* row = scores + (size_t)b * max_ctx;
  int32_t* orow = out + (size_t)b * topk;
  if (n <= topk) {
    for (int i = t; i < topk; i += kTkThreads) orow[i] = i < n ? i : -1;
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int need = topk;   // keys still to take among those matching prefix
  const uint32_t lt = (1u << lane) - 1u;
  if (n <= kTkThreads * kTkPer) {
    uint32_t key[kTkPer];
#pragma unroll
    for (int k = 0; k < kTkPer; ++k) {
      const int i = k * kTkThreads + t;
      key[k] = i < n ? order_key(row[i]) : 0u;
    }
    // three digits of 11, 11 and 10 bits: the top digit spans the sign,
    // the exponent and two mantissa bits, so keys of one magnitude still
    // spread over several bins (fewer colliding atomics than 8-bit digits)
    int eq_count = 0;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t dmask = pass == 2 ? 1023u : 2047u;
      hist[t] = 0;
      hist[t + 1024] = 0;
      __syncthreads();
      // one shared-memory atomic per key: with 11-bit digits the keys of a
      // warp spread over many bins, so same-address conflicts stay few
#pragma unroll
      for (int k = 0; k < kTkPer; ++k) {
        const bool in = k * kTkThreads + t < n && (key[k] & mask) == prefix;
        if (in) atomicAdd(&hist[(key[k] >> shift) & dmask], 1u);
      }
      __syncthreads();
      radix_pick2048(hist, need, sums, &s_digit, &s_need, &s_cnt);
      prefix |= s_digit << shift;
      mask |= dmask << shift;
      need = s_need;
      eq_count = s_cnt;
      __syncthreads();
    }
    unsigned selm[kTkPer];
    if (eq_count == need) {
      // every key equal to the selection is taken (the usual case)
#pragma unroll
      for (int k = 0; k < kTkPer; ++k)
        selm[k] = __ballot_sync(0xffffffffu, k * kTkThreads + t < n && key[k] >= prefix);
    } else {
      // ties: rank of each key equal to the selection among them, by position
      unsigned eqm[kTkPer];
#pragma unroll
      for (int k = 0; k < kTkPer; ++k) {
        eqm[k] = __ballot_sync(0xffffffffu, k * kTkThreads + t < n && key[k] == prefix);
        if (lane == 0) cnt[k * 32 + warp] = __popc(eqm[k]);
      }
      __syncthreads();
      if (t < 32) prefix256(cnt);
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kTkPer; ++k) {
        const bool valid = k * kTkThreads + t < n;
        const bool eq = (eqm[k] >> lane) & 1u;
        const int eq_rank = cnt[k * 32 + warp] + __popc(eqm[k] & lt);
        selm[k] = __ballot_sync(0xffffffffu, valid && (key[k] > prefix || (eq && eq_rank < need)));
      }
      __syncthreads();   // every eq rank read before cnt is reused
    }
#pragma unroll
    for (int k = 0; k < kTkPer; ++k)
      if (lane == 0) cnt[k * 32 + warp] = __popc(selm[k]);
    __syncthreads();
    if (t < 32) prefix256(cnt);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kTkPer; ++k) {
      if ((selm[k] >> lane) & 1u) {
        const int pos = cnt[k * 32 + warp] + __popc(selm[k] & lt);
        if (pos < topk) orow[pos] = k * kTkThreads + t;
      }
    }
    if (t == 0) grid_dep_launch();
    return;
  }
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (t < 256) hist[t] = 0;
    __syncthreads();
#pragma unroll 1
    for (int base = 0; base < n; base += kTkThreads) {
      const int i = base + t;
      const uint32_t key = i < n ? order_key(row[i]) : 0u;
      const bool in = i < n && (key & mask) == prefix;
      const uint32_t digit = (key >> shift) & 255u;
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned same = __match_any_sync(act, digit);
        if (lane == __ffs(same) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(same));
      }
    }
    __syncthreads();
    if (t < 32) radix_pick(hist, need, &s_digit, &s_need);
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    need = s_need;
    __syncthreads();
  }
  // prefix is now the topk-th largest key; take every larger key and the
  // first `need` (lowest positions) equal to it
  int written = 0, ties = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += kTkThreads) {
    const int i = base + t;
    const uint32_t key = i < n ? order_key(row[i]) : 0u;
    const bool gt = i < n && key > prefix;
    const bool eq = i < n && key == prefix;
    int eq_total, sel_total;
    const int eq_rank = block_prefix_count(eq, sums, &eq_total);
    const bool sel = gt || (eq && ties + eq_rank < need);
    const int pos = block_prefix_count(sel, sums, &sel_total);
    if (sel && written + pos < topk) orow[written + pos] = i;
    written += sel_total;
    ties += eq_total;
  }
  if (t == 0) grid_dep_launch();
}

// ------------------------------------------------------------------ host
static smla_status validate_indexer_shape(const smla_indexer_shape* s) {
  if (!s) return SMLA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535 || s->topk < 1 || s->topk > 65536 || s->reserved != 0)
    return SMLA_ERR_INVALID_ARG;
  if (s->max_ctx < 1 || s->max_ctx > (1 << 20)) return SMLA_ERR_INVALID_ARG;
  if (s->heads != kIxH || s->dim != kIxD || s->page_size != 64) return SMLA_ERR_UNSUPPORTED;
  if (s->pages_per_seq < 1 || (long long)s->pages_per_seq * 64 < s->max_ctx) return SMLA_ERR_INVALID_ARG;
  if (s->num_key_rows < 64 || s->num_key_rows % 64 != 0) return SMLA_ERR_INVALID_ARG;
  return SMLA_OK;
}

static cudaError_t launch_pdl(const void* kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kern, args);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (looked
// up once; null if the driver does not offer it)
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

static smla_status run_indexer_scores(const smla_indexer_shape* s, const void* q, const float* w, const void* k,
                                      const int32_t* page_table, const int32_t* ctx_len, float* scores,
                                      cudaStream_t stream) {
  static volatile int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SMLA_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(smla_indexer_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kIxSmemBytes) != cudaSuccess)
      return SMLA_ERR_CUDA;
    attr_done[dev] = 1;
  }
  IndexerParams prm;
  // the key cache as a tensor map (host-side encoding, no device call)
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return SMLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)kIxD, (cuuint64_t)s->num_key_rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kIxD * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&prm.kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return SMLA_ERR_CUDA;
  prm.q = static_cast<const uint8_t*>(q);
  prm.w = w;
  prm.k = static_cast<const uint8_t*>(k);
  prm.page_table = page_table;
  prm.ctx_len = ctx_len;
  prm.scores = scores;
  prm.max_ctx = s->max_ctx;
  prm.pages_per_seq = s->pages_per_seq;
  prm.num_rows = s->num_key_rows;
  void* args[] = {&prm};
  const dim3 grid((unsigned)((s->max_ctx + kIxTile - 1) / kIxTile), (unsigned)s->batch, 1);
  if (launch_pdl((const void*)smla_indexer_score_kernel, grid, dim3(kIxThreads), kIxSmemBytes, stream, args) !=
      cudaSuccess)
    return SMLA_ERR_CUDA;
  return SMLA_OK;
}

static smla_status run_indexer_topk(const smla_indexer_shape* s, const float* scores, const int32_t* ctx_len,
                                    int32_t* indices, cudaStream_t stream) {
  int max_ctx = s->max_ctx, topk = s->topk;
  void* args[] = {&scores, &ctx_len, &max_ctx, &topk, &indices};
  if (launch_pdl((const void*)smla_topk_kernel, dim3((unsigned)s->batch), dim3(kTkThreads), 0, stream, args) !=
      cudaSuccess)
    return SMLA_ERR_CUDA;
  return SMLA_OK;
}

}  // namespace smla

extern "C" {

smla_status sparse_mla_indexer_scores(const smla_indexer_shape* shape, const void* q, const float* w,
                                      const void* k_cache, const int32_t* page_table, const int32_t* ctx_len,
                                      float* scores, void* stream) {
  const smla_status st = smla::validate_indexer_shape(shape);
  if (st != SMLA_OK) return st;
  if (!q || !w || !k_cache || !page_table || !ctx_len || !scores) return SMLA_ERR_INVALID_ARG;
  if (!smla::aligned(q, 16) || !smla::aligned(k_cache, 16) || !smla::aligned(w, 4) ||
      !smla::aligned(page_table, 4) || !smla::aligned(ctx_len, 4) || !smla::aligned(scores, 4))
    return SMLA_ERR_INVALID_ARG;
  return smla::run_indexer_scores(shape, q, w, k_cache, page_table, ctx_len, scores,
                                  static_cast<cudaStream_t>(stream));
}

smla_status sparse_mla_indexer_topk(const smla_indexer_shape* shape, const float* scores, const int32_t* ctx_len,
                                    int32_t* indices, void* stream) {
  const smla_status st = smla::validate_indexer_shape(shape);
  if (st != SMLA_OK) return st;
  if (!scores || !ctx_len || !indices) return SMLA_ERR_INVALID_ARG;
  if (!smla::aligned(scores, 4) || !smla::aligned(ctx_len, 4) || !smla::aligned(indices, 4))
    return SMLA_ERR_INVALID_ARG;
  return smla::run_indexer_topk(shape, scores, ctx_len, indices, static_cast<cudaStream_t>(stream));
}

smla_status sparse_mla_indexer(const smla_indexer_shape* shape, const void* q, const float* w, const void* k_cache,
                               const int32_t* page_table, const int32_t* ctx_len, float* scores,
                               int32_t* indices, void* stream) {
  const smla_status st = smla::validate_indexer_shape(shape);
  if (st != SMLA_OK) return st;
  if (!indices || !smla::aligned(indices, 4)) return SMLA_ERR_INVALID_ARG;
  const smla_status a = sparse_mla_indexer_scores(shape, q, w, k_cache, page_table, ctx_len, scores, stream);
  if (a != SMLA_OK) return a;
  return sparse_mla_indexer_topk(shape, scores, ctx_len, indices, stream);
}

}  // extern "C"
