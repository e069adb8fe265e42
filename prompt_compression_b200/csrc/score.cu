// score.cu -- lookahead importance scoring on tcgen05 tensor cores.
//
// What it computes ("Draft-based Approximate Inference for LLMs", paper
// notes, section 关键设计):
//   SpecKV: for each KV head, the queries of the last n_window input tokens
//   and of the n_lookahead draft tokens (all g query heads of the GQA group)
//   attend causally to the input keys; the attention each prefix key gets,
//   summed over those queries, is its importance.
//   SpecPC: the same attention from the last W draft query positions, each
//   row weighted (weights fall towards older rows), averaged over queries and
//   over layers >= l_skip, then maximised over query heads.
//
// The column sum of a row-normalised softmax needs each row's normaliser
// before any column can be summed, so the work is two passes over Q.K^T:
//   pass 1 (MODE_LSE): lane = query row, columns = keys; online max / sum of
//                      exp2 gives lse2[row] = log2 sum_j 2^(c2 * q.k_j).
//   pass 2 (MODE_COLSUM / MODE_COLSUM_PC): lane = key, columns = query rows;
//                      sum_rows 2^(c2 * q.k - lse2[row]) is the key's score.
// Both passes share one persistent, warp-specialised kernel:
//   warp 16   : TMA producer: an item's two A tiles once per segment, the
//               segment's row offsets (-lse2, one bulk copy), B tiles streamed
//   warp 17   : TMEM allocator + single-thread UMMA issuer (128 x N x 16 bf16)
//   warps 0-15: epilogue; warp w owns TMEM lane quadrant w % 4 of A tile w / 8
//               and one column half of every accumulator stage (four warps
//               per SM sub-partition hide the latency of the exp2 chains); the
//               two halves of a lane are merged in shared memory per item.
// TMEM (512 columns):
//   pass 1: the item's two A tiles (copied from shared memory with
//           tcgen05.cp, so the UMMAs read only B from shared memory) and three
//           128-column fp32 accumulator buffers that the two tiles rotate
//           through; its items are long, so refilling A is rare.
//   pass 2: A changes every few steps, so it is read from (double-buffered)
//           shared memory and four 128-column accumulator buffers rotate.
// The epilogues use packed fp32x2 math; a share of the exponentials runs on
// the FMA pipe (exp2_poly.cuh) and the rest on the MUFU.
// No atomics: every output element is reduced by exactly one thread in a
// fixed order, so results are bitwise reproducible.
#include <cuda_bf16.h>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "score.cuh"

namespace spk {

SPK_ERROR_READER(device_errors_score)

namespace {

// 16 epilogue warps (4 per SM sub-partition, to hide latency), then the
// producer warp and the MMA warp.
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 18 * 32;

// Exponential pairs p with (p & 7) < POLY_OF_8 run on the FMA pipe
// (exp2_poly.cuh), the others on the MUFU (16 exponentials per clock per SM).
// The board runs at its power cap during these passes, where FMA-pipe
// polynomials cost clock; the measured best shares are 1 of 8 for the row
// pass and 2 of 8 for the column passes.
constexpr int kPolyRowPass = 1;
constexpr int kPolyPairsOf8 = 2;
constexpr int kPolyPcPairsOf8 = 1;   // the SpecPC column pass (measured best)

template <int MODE, int D>
struct Cfg {
  static constexpr int kTileBytes = 128 * D * 2;          // 128 rows x D bf16
  static constexpr int kAtoms = D / 64;                    // 128-byte swizzle atoms along K
  // The SpecPC column pass at head_dim 128 keeps one A stage: two stages
  // (128 KB) next to the B ring and the per-head sums would exceed 227 KB.
  static constexpr int kAStages = (MODE == MODE_LSE || (MODE == MODE_COLSUM_PC && D == 128)) ? 1 : 2;
  static constexpr int kBStages = (MODE == MODE_LSE) ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 4);
  static constexpr int kABytes = 2 * kTileBytes;
  static constexpr int kSmemA = kAStages * kABytes;
  // column passes: each B stage also holds its tile's row-offset block, and a
  // block of ones (the keys' side of the offset K-step) follows the stages
  static constexpr int kOffBytes = (MODE == MODE_LSE) ? 0 : kOffBlockBytes;
  static constexpr int kBStageBytes = kTileBytes + kOffBytes;
  static constexpr int kSmemB = kBStages * kBStageBytes;
  static constexpr int kOnesBytes = kOffBytes;
  static constexpr int kAccFloats = (MODE == MODE_COLSUM_PC) ? 2 * kHeadsMax * 256 : 0;
  static constexpr int kSmemBytes = 1024 + kSmemA + kSmemB + kOnesBytes + 4 * kAccFloats;
  static_assert(kBStageBytes % 1024 == 0, "B stages keep the 1024-byte alignment of the swizzled tiles");
  static_assert(kSmemBytes <= 227 * 1024 - 4096, "dynamic shared memory (plus the static part) fits one CTA");
  // Pass 1 items are long (all keys of a unit): its A tiles live in TMEM and
  // the UMMAs read only B from shared memory; three accumulator buffers fill
  // the rest of TMEM.  The column passes change A every few steps: A stays in
  // (double-buffered) shared memory and four accumulator buffers rotate.
  static constexpr bool kATmem = (MODE == MODE_LSE);
  static constexpr uint32_t kNumAcc = kATmem ? 3 : 4;
};

// n / R and n % R for 0 <= n <= 4096 (rows of a unit, R <= 2048) by a
// multiply-high with ceil(2^32 / R): n * R < 2^32 keeps the quotient exact.
__device__ __forceinline__ int div_R(const ScoreParams& p, int n) {
  return p.R == 1 ? n : static_cast<int>(__umulhi(static_cast<uint32_t>(n), p.R_mul));
}
__device__ __forceinline__ int mod_R(const ScoreParams& p, int n) { return n - div_R(p, n) * p.R; }

// Error sites: mode * 100 + role * 10 + barrier.
__device__ __forceinline__ int site(int mode, int role, int which) { return mode * 100 + role * 10 + which; }

// Segments of an item: SpecPC walks the (KV head, layer) segments of its
// batch element, split into p.seg_groups contiguous groups (item =
// (key block) * seg_groups + group); the other modes have one segment.
__device__ __forceinline__ int seg_begin(const ScoreParams& p, int mode, int item) {
  if (mode != MODE_COLSUM_PC) return 0;
  const int nseg = p.hkv * p.layers_used;
  return static_cast<int>(static_cast<long long>(item % p.seg_groups) * nseg / p.seg_groups);
}
__device__ __forceinline__ int seg_end(const ScoreParams& p, int mode, int item) {
  if (mode != MODE_COLSUM_PC) return 1;
  const int nseg = p.hkv * p.layers_used;
  return static_cast<int>(static_cast<long long>(item % p.seg_groups + 1) * nseg / p.seg_groups);
}

// (item, segment) -> unit, its 3-D tensor coordinate, first A row.
__device__ __forceinline__ void decode(const ScoreParams& p, int mode, int item, int seg, int& u, int& tc,
                                       int& a_row0) {
  if (mode == MODE_COLSUM_PC) {
    const int blk = item / p.seg_groups;
    const int b = blk / p.n_blocks;
    const int h = seg / p.layers_used, lu = seg % p.layers_used;
    u = (b * p.layers_used + lu) * p.hkv + h;
    a_row0 = (blk % p.n_blocks) * 256;
  } else {
    u = item / p.n_blocks;
    a_row0 = (item % p.n_blocks) * 256;
  }
  const int h = u % p.hkv;
  const int rest = u / p.hkv;
  const int lu = rest % p.layers_used;
  const int b = rest / p.layers_used;
  tc = (b * p.layers_total + p.l_skip + lu) * p.hkv + h;
}

__device__ __forceinline__ int b_tiles(const ScoreParams& p, int mode) {
  return mode == MODE_LSE ? (p.n_in + 127) / 128 : (p.rows + 127) / 128;
}

// A tile t is worth computing: LSE -> it holds query rows; column sums -> it
// holds keys that are written out.
__device__ __forceinline__ bool a_tile_active(const ScoreParams& p, int mode, int a_row0, int t) {
  return mode == MODE_LSE ? (a_row0 + 128 * t < p.rows) : (a_row0 + 128 * t < p.n_cols);
}

// Columns of B chunk bt in a column-sum pass: valid rows rounded up to 32 so
// that every TMEM column the epilogue reads was written by this MMA.
__device__ __forceinline__ int chunk_cols(const ScoreParams& p, int bt) {
  const int left = p.rows - bt * 128;
  return left >= 128 ? 128 : ((left + 31) & ~31);
}

// ---------------------------------------------------------------------------
// pass-1 epilogue: online log2-sum-exp2 over 64 keys (jb .. jb+63) of one row
// ---------------------------------------------------------------------------
// Mask-free core: every one of the 64 logits x is visible (or already -inf).
template <int POLY_OF_8>
__device__ __forceinline__ void lse_core64(const float (&x)[64], float c2, float& m, float& l) {
  float a0 = fmaxf(x[0], x[1]), a1 = fmaxf(x[2], x[3]), a2 = fmaxf(x[4], x[5]), a3 = fmaxf(x[6], x[7]);
#pragma unroll
  for (int k = 8; k < 64; k += 8) {
    a0 = max3f(a0, x[k + 0], x[k + 1]);
    a1 = max3f(a1, x[k + 2], x[k + 3]);
    a2 = max3f(a2, x[k + 4], x[k + 5]);
    a3 = max3f(a3, x[k + 6], x[k + 7]);
  }
  const float mx = max3f(a0, a1, fmaxf(a2, a3));
  const float mn = fmaxf(m, mx * c2);
  const float2 c2v = f2(c2, c2), nm = f2(-mn, -mn);
  float2 s[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float2 t = __ffma2_rn(f2(x[2 * p], x[2 * p + 1]), c2v, nm);
    const float2 e = ((p & 7) < POLY_OF_8) ? exp2_fma_pair(t) : exp2_mufu_pair(t);
    s[p & 3] = __fadd2_rn(s[p & 3], e);
  }
  const float2 s01 = __fadd2_rn(__fadd2_rn(s[0], s[1]), __fadd2_rn(s[2], s[3]));
  if (mn > m) l *= ex2_approx(m - mn);    // first update: m = -inf, ex2(-inf) = 0
  l += s01.x + s01.y;
  m = mn;
}

// Keys jb .. jb+63 of a row that sees keys [0, c).  Tiles that straddle c
// take a separate masked copy, so the common path carries no per-key
// compare/select.
template <int POLY_OF_8>
__device__ __forceinline__ void lse_update64(const uint32_t (&va)[32], const uint32_t (&vb)[32], int jb, int c,
                                             float c2, float& m, float& l) {
  if (jb >= c) return;
  float x[64];
  if (jb + 64 <= c) {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      x[k] = __uint_as_float(va[k]);
      x[32 + k] = __uint_as_float(vb[k]);
    }
    lse_core64<POLY_OF_8>(x, c2, m, l);
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      x[k] = (jb + k < c) ? __uint_as_float(va[k]) : -INFINITY;
      x[32 + k] = (jb + 32 + k < c) ? __uint_as_float(vb[k]) : -INFINITY;
    }
    lse_core64<POLY_OF_8>(x, c2, m, l);
  }
}

// ---------------------------------------------------------------------------
// pass-2 epilogue: s += 2^(c2 x) over 32 rows, where the accumulator x
// already holds q.k - lse2[row] / c2 (the offset K-step)
// ---------------------------------------------------------------------------
// CUT: the first `cut` (0..32) of the 32 rows cannot see this thread's key;
// their exponent becomes -inf (MUFU: exactly 0; FMA pipe: 2^-126, far below
// the rounding of any sum it joins).  With cut = 0 the arithmetic, and so the
// result, is bit for bit that of the unmasked form.
template <int POLY_OF_8, bool CUT = false>
__device__ __forceinline__ void colsum32(const uint32_t (&v)[32], float c2, float2 (&s)[4], int cut = 0) {
  const float2 c2v = f2(c2, c2);
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    float2 t = __fmul2_rn(f2(__uint_as_float(v[2 * p]), __uint_as_float(v[2 * p + 1])), c2v);
    if (CUT) {
      if (2 * p + 0 < cut) t.x = -INFINITY;
      if (2 * p + 1 < cut) t.y = -INFINITY;
    }
    const float2 e = ((p & 7) < POLY_OF_8) ? exp2_fma_pair(t) : exp2_mufu_pair(t);
    s[p & 3] = __fadd2_rn(s[p & 3], e);
  }
}

// Row r (0..127) of a row-offset block (layout: kOffBlockBytes): v split
// into three bf16 terms, h1 = bf16(v), h2 = bf16(v - h1), h3 = bf16(v - h1 - h2).
__device__ __forceinline__ void store_offset_row(uint8_t* block, int r, float v) {
  const __nv_bfloat16 h1 = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h1);
  const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(h2);
  const __nv_bfloat16 h3 = __float2bfloat16_rn(r2);
  const uint32_t w0 = static_cast<uint32_t>(__bfloat16_as_ushort(h1)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h2)) << 16);
  const uint32_t w1 = static_cast<uint32_t>(__bfloat16_as_ushort(h3));
  uint8_t* row = block + (r >> 3) * 256 + (r & 7) * 16;
  *reinterpret_cast<uint4*>(row) = make_uint4(w0, w1, 0u, 0u);
  *reinterpret_cast<uint4*>(row + 128) = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ float fold(const float2 (&s)[4]) {
  const float2 t = __fadd2_rn(__fadd2_rn(s[0], s[1]), __fadd2_rn(s[2], s[3]));
  return t.x + t.y;
}

// For a key j that some rows cannot see: row n (head-local i = n % R) sees
// key j only if j < c0 + i.  nb is the first row of the 32.
__device__ __forceinline__ float colsum32_masked(const uint32_t (&v)[32], int i, float c2, int j, int c0, int R) {
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    if (j < c0 + i) s += ex2_approx(__uint_as_float(v[k]) * c2);
    if (++i == R) i = 0;
  }
  return s;
}

}  // namespace

// 18 warps: two SM sub-partitions hold 5 warps, so at most 96 registers per
// thread fit their 16,384-register files.
template <int MODE, int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                 const ScoreParams p) {
  using C = Cfg<MODE, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const A_s = smem;
  uint8_t* const B_s = smem + C::kSmemA;
  uint8_t* const ones_s = B_s + C::kSmemB;                                  // column passes: offset K-step, keys' side
  float* const acc_s = reinterpret_cast<float*>(ones_s + C::kOnesBytes);   // SpecPC: [2][kHeadsMax][256]

  __shared__ __align__(8) uint64_t a_full[2], a_empty[2], b_full[8], b_empty[8], acc_full[4], acc_empty[4],
      mrg_full[2], mrg_empty[2], seg_done, done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  __shared__ float wsum_s[kThreads / 32];
  __shared__ float xm_s[256], xl_s[256];   // column-half merge of per-row / per-key partials

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kAStages; ++s) { mbar_init(&a_full[s], 1); mbar_init(&a_empty[s], 1); }
    for (int s = 0; s < C::kBStages; ++s) { mbar_init(&b_full[s], 1); mbar_init(&b_empty[s], 1); }
    for (int s = 0; s < (int)C::kNumAcc; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], kEpiWarps / 2); }
    mbar_init(&seg_done, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&mrg_full[s], kEpiWarps / 2); mbar_init(&mrg_empty[s], kEpiWarps / 2); }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_map(&amap);
    tma_prefetch_map(&bmap);
  }
  if (MODE == MODE_COLSUM_PC && threadIdx.x < kEpiThreads)
    for (int n = threadIdx.x; n < C::kAccFloats; n += kEpiThreads) acc_s[n] = 0.f;
  if (MODE != MODE_LSE && threadIdx.x < 256) {
    // ones block: every key row has K-chunk 0 = (1, 1, 1, 0 x 5), chunk 1 = 0
    // (no-swizzle K-major layout of kOffBlockBytes); made visible to the
    // tensor pipe (async proxy) before the barrier below
    const int r = threadIdx.x >> 1, c = threadIdx.x & 1;
    const uint32_t one = 0x3F80u;   // bf16 1.0
    const uint4 val = c == 0 ? make_uint4(one | (one << 16), one, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(ones_s + (r >> 3) * 256 + c * 128 + (r & 7) * 16) = val;
    fence_proxy_async_smem();
  }
  // Row-weight normaliser for SpecPC pass 1: log2(sum_i w_i * (L - l_skip)).
  float log2_norm = 0.f;
  if (MODE == MODE_LSE && p.row_weights != nullptr) {
    float s = 0.f;
    for (int i = threadIdx.x; i < p.R; i += kThreads) s += p.row_weights[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wsum_s[warp] = s;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (MODE == MODE_LSE && p.row_weights != nullptr) {
    float s = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) s += wsum_s[w];
    log2_norm = log2f(s * static_cast<float>(p.layers_used));
  }
  const uint32_t tmem_base = tmem_holder;
  volatile int* abort_v = &abort_flag;
  const int nb = b_tiles(p, MODE);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t a_stage = 0, a_phase = 0, b_stage = 0, b_phase = 0;
      int a_last[2] = {-1, -1};
      int b_last[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
      int seg_count = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        for (int seg = seg_begin(p, MODE, item); ok && seg < seg_end(p, MODE, item); ++seg, ++seg_count) {
          int u, tc, a_row0;
          decode(p, MODE, item, seg, u, tc, a_row0);
          if (!(ok = mbar_wait(&a_empty[a_stage], a_phase ^ 1, abort_v, site(MODE, 0, 0)))) break;
          mbar_arrive_expect_tx(&a_full[a_stage], C::kABytes);
          uint8_t* dst = A_s + a_stage * C::kABytes;
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int a = 0; a < C::kAtoms; ++a)
              tma_load_3d(dst + t * C::kTileBytes + a * 16384, &amap, &a_full[a_stage], a * 64, a_row0 + 128 * t,
                          tc);
          a_last[a_stage] = static_cast<int>(a_phase);
          if (++a_stage == C::kAStages) { a_stage = 0; a_phase ^= 1; }
          for (int bt = 0; bt < nb; ++bt) {
            if (!(ok = mbar_wait(&b_empty[b_stage], b_phase ^ 1, abort_v, site(MODE, 0, 1)))) break;
            mbar_arrive_expect_tx(&b_full[b_stage], C::kBStageBytes);
            uint8_t* bdst = B_s + b_stage * C::kBStageBytes;
#pragma unroll
            for (int a = 0; a < C::kAtoms; ++a)
              tma_load_3d(bdst + a * 16384, &bmap, &b_full[b_stage], a * 64, bt * 128, tc);
            if (MODE != MODE_LSE)   // this tile's row-offset block, written by pass 1
              bulk_load(bdst + C::kTileBytes,
                        p.off_blocks + (static_cast<size_t>(u) * p.off_tiles + bt) * kOffBlockBytes,
                        kOffBlockBytes, &b_full[b_stage]);
            b_last[b_stage] = static_cast<int>(b_phase);
            if (++b_stage == C::kBStages) { b_stage = 0; b_phase ^= 1; }
          }
        }
      }
      if (!ok) {
        // unwind: let every copy this thread issued land before the CTA exits
        // (these waits ignore the abort flag but are still time-bounded)
        volatile int never = 0;
        for (int s = 0; s < C::kAStages; ++s)
          if (a_last[s] >= 0) mbar_wait(&a_full[s], a_last[s], &never, site(MODE, 0, 7), 100000000ull);
        for (int s = 0; s < C::kBStages; ++s)
          if (b_last[s] >= 0) mbar_wait(&b_full[s], b_last[s], &never, site(MODE, 0, 8), 100000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ UMMA issuer
    // TMEM columns: accumulator buffers at 128 * b; with A in TMEM (pass 1)
    // the two A tiles sit at 384 + t * D/2 (D/2 32-bit columns hold a 128 x D
    // bf16 tile).  Step k of tile t accumulates into buffer (2k + t) % kNumAcc,
    // its ((2k + t) / kNumAcc)-th use.
    if (lane == 0) {
      uint32_t a_stage = 0, a_phase = 0, b_stage = 0, b_phase = 0;
      uint32_t step = 0;           // accumulator steps issued by this CTA
      uint32_t segs = 0;           // segments started by this CTA
      bool ok = true;
      const uint32_t a_tmem0 = tmem_base + 384;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        for (int seg = seg_begin(p, MODE, item); ok && seg < seg_end(p, MODE, item); ++seg, ++segs) {
          int u, tc, a_row0;
          decode(p, MODE, item, seg, u, tc, a_row0);
          const bool act0 = a_tile_active(p, MODE, a_row0, 0);
          const bool act1 = a_tile_active(p, MODE, a_row0, 1);
          if (!(ok = mbar_wait(&a_full[a_stage], a_phase, abort_v, site(MODE, 1, 0)))) break;
          const uint64_t a_sdesc = sw128_kmajor_desc(smem_u32(A_s + a_stage * C::kABytes));
          if (C::kATmem) {
            // the previous segment's UMMAs must have read the TMEM A tiles
            if (segs > 0 && !(ok = mbar_wait(&seg_done, (segs - 1) & 1, abort_v, site(MODE, 1, 3)))) break;
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!(t == 0 ? act0 : act1)) continue;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t koff = ((t * C::kTileBytes) + (kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                tmem_cp_128x256b(a_tmem0 + t * (D / 2) + kk * 8, a_sdesc + koff);
              }
            }
            umma_commit(&a_empty[a_stage]);   // the shared-memory A stage is free once copied
          } else {
            tc_fence_after();
          }
          for (int bt = 0; bt < nb; ++bt, ++step) {
            if (!(ok = mbar_wait(&b_full[b_stage], b_phase, abort_v, site(MODE, 1, 1)))) break;
            const int n = (MODE == MODE_LSE) ? 128 : chunk_cols(p, bt);
            const uint32_t idesc = idesc_bf16_f32(128, n);
            const uint64_t b_desc0 = sw128_kmajor_desc(smem_u32(B_s + b_stage * C::kBStageBytes));
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const uint32_t use = 2 * step + t;
              const uint32_t buf = use % C::kNumAcc;
              if (!(ok = mbar_wait(&acc_empty[buf], ((use / C::kNumAcc) & 1) ^ 1, abort_v, site(MODE, 1, 2))))
                break;
              tc_fence_after();
              if (t == 0 ? act0 : act1) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const uint64_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                  if (C::kATmem)
                    umma_bf16_ts(tmem_base + buf * 128, a_tmem0 + t * (D / 2) + kk * 8, b_desc0 + koff, idesc,
                                 kk > 0 ? 1u : 0u);
                  else
                    umma_bf16_ss(tmem_base + buf * 128, a_sdesc + ((t * C::kTileBytes) >> 4) + koff, b_desc0 + koff,
                                 idesc, kk > 0 ? 1u : 0u);
                }
                if (MODE != MODE_LSE) {
                  // offset K-step: ones (keys) x (h1, h2, h3) (query rows) adds
                  // -lse2[row] / c2 to every logit of the row
                  umma_bf16_ss(tmem_base + buf * 128, nosw_kmajor_desc(smem_u32(ones_s), 128, 256),
                               nosw_kmajor_desc(smem_u32(B_s + b_stage * C::kBStageBytes + C::kTileBytes), 128, 256),
                               idesc, 1u);
                }
              }
              umma_commit(&acc_full[buf]);
            }
            if (!ok) break;
            umma_commit(&b_empty[b_stage]);
            if (++b_stage == C::kBStages) { b_stage = 0; b_phase ^= 1; }
          }
          if (!ok) break;
          if (C::kATmem) {
            umma_commit(&seg_done);
          } else {
            umma_commit(&a_empty[a_stage]);   // this segment's UMMAs have read the A stage
          }
          if (++a_stage == C::kAStages) { a_stage = 0; a_phase ^= 1; }
        }
      }
      // every UMMA this thread issued has finished before TMEM is freed
      umma_commit(&done_bar);
      volatile int never = 0;
      mbar_wait(&done_bar, 0, &never, site(MODE, 1, 9), 100000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: A tile t = w / 8, column half hc = (w / 4) % 2 of every
    // accumulator stage, TMEM lane quadrant q = w % 4.  The two column halves
    // of a lane are merged through shared memory at the end of each item.
    const int t = warp >> 3;
    const int hc = (warp >> 2) & 1;
    const int q = warp & 3;
    const int r = t * 128 + q * 32 + lane;   // A row within the item
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t step = 0;               // accumulator steps consumed (same count as the MMA thread)
    int seg_count = 0, items_done = 0;
    bool ok = true;
    uint32_t acc_buf = t;            // buffer of this tile at the current step: (2 * step + t) % kNumAcc

    auto wait_acc = [&](int which) -> bool {
      const uint32_t use = 2 * step + t;
      bool w = mbar_wait(&acc_full[acc_buf], (use / C::kNumAcc) & 1, abort_v, site(MODE, 2, which));
      w = __all_sync(0xffffffffu, w);
      if (w) tc_fence_after();
      return w;
    };
    auto release_acc = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc_buf]);
    };
    auto next_acc = [&]() {
      ++step;
      acc_buf = (2 * step + t) % C::kNumAcc;
    };
    auto wait_uniform = [&](uint64_t* bar, uint32_t parity, int which) -> bool {
      bool w = mbar_wait(bar, parity, abort_v, site(MODE, 3, which));
      return __all_sync(0xffffffffu, w);
    };
    auto arrive_warp = [&](uint64_t* bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // SpecKV column sums, first half: the item whose second-half partial is
    // still to be added, and the step that adds it and stores the total
    float pend_part = 0.f;
    int pend_u = 0, pend_row0 = 0;
    auto colsum_flush = [&](int n) -> bool {
      const int slot = n & 1;
      if (!wait_uniform(&mrg_full[slot], (n >> 1) & 1, 1)) return false;
      const float total = pend_part + (slot ? xl_s : xm_s)[r];
      arrive_warp(&mrg_empty[slot]);
      const int j = pend_row0 + r;
      if (a_tile_active(p, MODE, pend_row0, t)) {
        if (j < p.n_pre) p.out0[static_cast<size_t>(pend_u) * p.n_pre + j] = total;
        else if (j < p.n_cols && p.out1 != nullptr)
          p.out1[static_cast<size_t>(pend_u) * (p.n_in - p.n_pre) + (j - p.n_pre)] = total;
      }
      return true;
    };

    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++items_done) {
      // the second column half may not touch the merge buffers (or, for
      // SpecPC, its head sums) until the first half has consumed the last item's
      if (MODE != MODE_COLSUM && hc == 1 && items_done > 0 &&
          !(ok = wait_uniform(&mrg_empty[0], (items_done - 1) & 1, 0)))
        break;
      float2 sacc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};   // SpecKV column sum
      float acc_masked = 0.f;
      float m = -INFINITY, l = 0.f;                                                 // pass-1 row state
      int item_u = 0, item_row0 = 0;
      for (int seg = seg_begin(p, MODE, item); ok && seg < seg_end(p, MODE, item); ++seg, ++seg_count) {
        int u, tc, a_row0;
        decode(p, MODE, item, seg, u, tc, a_row0);
        item_u = u;
        item_row0 = a_row0;
        const bool active = a_tile_active(p, MODE, a_row0, t);
        if (MODE == MODE_LSE) {
          const int row = a_row0 + r;
          const bool row_ok = active && row < p.rows;
          const int c = min(p.n_in, p.c0 + (row_ok ? mod_R(p, row) : 0));
          for (int bt = 0; bt < nb; ++bt) {
            if (!(ok = wait_acc(0))) break;
            if (active) {
              const uint32_t taddr = tbase + acc_buf * 128 + hc * 64;
              uint32_t va[32], vb[32];
              tmem_ld32(taddr, va);
              tmem_ld32(taddr + 32, vb);
              tmem_ld_wait2(va, vb);
              release_acc();
              if (row_ok) lse_update64<kPolyRowPass>(va, vb, bt * 128 + hc * 64, c, p.c2, m, l);
            } else {
              release_acc();
            }
            next_acc();
          }
        } else {
          const int j = a_row0 + r;              // this thread's key
          const bool masked_key = j >= p.c0;     // some rows cannot see it
          // Rows with head-local index i <= j - c0 cannot see key j.  The
          // warp's keys are consecutive, so per 32-row group (that stays in
          // one head) the warp can tell whether no row, every row or a
          // leading part of the rows is masked for its keys.
          // (Only m_lane stays live through the loop; the warp-wide facts are
          // recomputed per group, which costs a vote in the common case.)
          const int m_lane = masked_key ? j - p.c0 : -1;
          const bool warp_masked = __any_sync(0xffffffffu, m_lane >= 0);   // some key of the warp is masked
          // 0: no row masked, 1: every row masked, 2: leading rows masked,
          // 3: the group wraps into the next head (per-row test)
          auto mask_class = [&](int nb0) -> int {
            if (!__any_sync(0xffffffffu, m_lane >= 0)) return 0;
            const int i0 = mod_R(p, nb0);
            if (i0 + 32 > p.R) return 3;
            if (__reduce_max_sync(0xffffffffu, m_lane) < i0) return 0;
            if (__reduce_min_sync(0xffffffffu, m_lane) >= i0 + 31) return 1;
            return 2;
          };
          const int gh = div_R(p, p.rows);       // query heads of the unit
          const int head0 = (seg / p.layers_used) * gh;   // SpecPC: first query head of this KV head
          float seg_sum = 0.f;
          int cur_head = -1;
          float* my_acc = acc_s + hc * kHeadsMax * 256;
          for (int bt = 0; bt < nb; ++bt) {
            if (!(ok = wait_acc(1))) break;
            // this warp's columns of the chunk: the first half takes ncols/2
            // rounded up to 32, the second the rest (possibly none, and then it
            // only releases the buffer)
            const int ncols = chunk_cols(p, bt);
            const int half = ((ncols >> 1) + 31) & ~31;
            const int col0 = hc == 0 ? 0 : half;
            const int width = active ? (hc == 0 ? half : ncols - half) : 0;
            auto process32 = [&](const uint32_t (&v)[32], int nb0) {
              if (MODE == MODE_COLSUM) {
                const int mc = mask_class(nb0);
                if (mc == 0) {
                  colsum32<kPolyPairsOf8>(v, p.c2, sacc);
                } else if (mc == 2) {
                  colsum32<kPolyPairsOf8, true>(v, p.c2, sacc, min(32, max(0, m_lane - mod_R(p, nb0) + 1)));
                } else if (mc == 3) {
                  if (masked_key) acc_masked += colsum32_masked(v, mod_R(p, nb0), p.c2, j, p.c0, p.R);
                  else colsum32<kPolyPairsOf8>(v, p.c2, sacc);
                }
              } else {
                // SpecPC: rows of one query head are contiguous (R = W rows);
                // rows >= p.rows are padding and belong to no head
                const int h0 = div_R(p, nb0), h1 = div_R(p, nb0 + 31);
                if (h0 >= gh) {
                  // the whole group is padding
                } else if (h0 == h1) {
                  if (h0 != cur_head) {
                    if (cur_head >= 0) my_acc[(head0 + cur_head) * 256 + r] += seg_sum;
                    cur_head = h0;
                    seg_sum = 0.f;
                  }
                  // h0 == h1: the group stays in one head
                  const int mc = mask_class(nb0);
                  if (mc == 0) {
                    float2 gs[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
                    colsum32<kPolyPcPairsOf8>(v, p.c2, gs);
                    seg_sum += fold(gs);
                  } else if (mc == 2) {
                    float2 gs[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
                    colsum32<kPolyPcPairsOf8, true>(v, p.c2, gs, min(32, max(0, m_lane - mod_R(p, nb0) + 1)));
                    seg_sum += fold(gs);
                  }
                } else {
                  // a 32-row group that straddles two query heads
                  int i = mod_R(p, nb0);
                  for (int k = 0; k < 32; ++k) {
                    const int n = nb0 + k;
                    if (n >= p.rows) break;
                    const int hh = div_R(p, n);
                    if (hh != cur_head) {
                      if (cur_head >= 0) my_acc[(head0 + cur_head) * 256 + r] += seg_sum;
                      cur_head = hh;
                      seg_sum = 0.f;
                    }
                    if (!masked_key || j < p.c0 + i)
                      seg_sum += ex2_approx(__uint_as_float(v[k]) * p.c2);
                    if (++i == p.R) i = 0;
                  }
                }
              }
            };
            // 32 columns per TMEM wait keeps the live registers within budget
            const uint32_t taddr = tbase + acc_buf * 128 + col0;
            if (width == 0) release_acc();
            if (MODE == MODE_COLSUM_PC && width > 0 && !warp_masked) {
              // SpecPC, no key of the warp masked for any row: when the
              // warp's columns are real rows of one query head, one head
              // switch and one fold for all of them
              const int nb0 = bt * 128 + col0;
              const int h0 = div_R(p, nb0);
              if (nb0 + width <= p.rows && h0 == div_R(p, nb0 + width - 1)) {
                if (h0 != cur_head) {
                  if (cur_head >= 0) my_acc[(head0 + cur_head) * 256 + r] += seg_sum;
                  cur_head = h0;
                  seg_sum = 0.f;
                }
                float2 gs[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
                for (int g = 0; g < width; g += 32) {
                  uint32_t v[32];
                  __syncwarp();
                  tmem_ld32(taddr + g, v);
                  tmem_ld_wait(v);
                  if (g + 32 >= width) release_acc();
                  colsum32<kPolyPcPairsOf8>(v, p.c2, gs);
                }
                seg_sum += fold(gs);
                next_acc();
                continue;
              }
            }
            for (int g = 0; g < width; g += 32) {
              uint32_t v[32];
              __syncwarp();
              tmem_ld32(taddr + g, v);
              tmem_ld_wait(v);
              if (g + 32 >= width) release_acc();
              process32(v, bt * 128 + col0 + g);
            }
            next_acc();
          }
          if (MODE == MODE_COLSUM_PC && ok && active && cur_head >= 0)
            my_acc[(head0 + cur_head) * 256 + r] += seg_sum;
        }
      }
      if (!ok) break;

      // ---- merge the two column halves and write this item's outputs
      if (MODE == MODE_LSE) {
        if (hc == 1) {
          xm_s[r] = m;
          xl_s[r] = l;
          arrive_warp(&mrg_full[0]);
        } else {
          if (!(ok = wait_uniform(&mrg_full[0], items_done & 1, 1))) break;
          const float m1 = xm_s[r], l1 = xl_s[r];
          arrive_warp(&mrg_empty[0]);
          const int row = item_row0 + r;
          if (a_tile_active(p, MODE, item_row0, t)) {
            float out = 0.f;
            bool live = row < p.rows;   // a row that contributes to the column sums
            if (live) {
              const float M = fmaxf(m, m1);
              const float L = l * ex2_approx(m - M) + l1 * ex2_approx(m1 - M);
              out = M + lg2_approx(L);
              if (p.row_weights != nullptr) {
                // weight w_i folds in as -log2(w_i); a row of weight 0 adds
                // nothing and takes the padding offset (log2(0) = -inf would
                // turn the three-term split into NaN)
                const float w = p.row_weights[mod_R(p, row)];
                if (w > 0.f) out += log2_norm - log2f(w);
                else live = false;
              }
            }
            if (p.off_blocks != nullptr) {
              if (row < p.off_tiles * 128)
                store_offset_row(p.off_blocks + (static_cast<size_t>(item_u) * p.off_tiles + row / 128) * kOffBlockBytes,
                                 row & 127, live ? -out / p.c2 : -1e30f);
            } else if (row < p.rows) {
              p.lse2[static_cast<size_t>(item_u) * p.lse_stride + row] = out;
            }
          }
        }
      } else if (MODE == MODE_COLSUM) {
        // The halves hand over through two slots, and the first half adds
        // item n's partials at the end of item n + 1: by then the second half
        // has long finished item n, so neither half waits for the other.
        const float part = fold(sacc) + acc_masked;
        const int slot = items_done & 1;
        if (hc == 1) {
          if (items_done >= 2 && !(ok = wait_uniform(&mrg_empty[slot], ((items_done - 2) >> 1) & 1, 0))) break;
          (slot ? xl_s : xm_s)[r] = part;
          arrive_warp(&mrg_full[slot]);
        } else {
          if (items_done >= 1 && !(ok = colsum_flush(items_done - 1))) break;
          pend_part = part;
          pend_u = item_u;
          pend_row0 = item_row0;
        }
      } else {
        // SpecPC: both halves' per-head sums are complete; max over query heads
        if (hc == 1) {
          arrive_warp(&mrg_full[0]);
        } else {
          if (!(ok = wait_uniform(&mrg_full[0], items_done & 1, 1))) break;
          const int hq = div_R(p, p.rows) * p.hkv;
          const int blk = item / p.seg_groups;
          if (p.seg_groups == 1) {
            float best = -INFINITY;
            for (int qh = 0; qh < hq; ++qh) {
              float* a0 = acc_s + qh * 256 + r;
              float* a1 = acc_s + (kHeadsMax + qh) * 256 + r;
              best = fmaxf(best, *a0 + *a1);
              *a0 = 0.f;
              *a1 = 0.f;
            }
            arrive_warp(&mrg_empty[0]);
            const int b = blk / p.n_blocks;
            const int j = (blk % p.n_blocks) * 256 + r;
            if (j < p.n_cols) p.out0[static_cast<size_t>(b) * p.n_in + j] = best;
          } else {
            // this group's per-head partial sums; specpc_merge adds the
            // groups in order and takes the head max
            float* part = p.part + static_cast<size_t>(item) * hq * 256 + r;
            for (int qh = 0; qh < hq; ++qh) {
              float* a0 = acc_s + qh * 256 + r;
              float* a1 = acc_s + (kHeadsMax + qh) * 256 + r;
              part[qh * 256] = *a0 + *a1;
              *a0 = 0.f;
              *a1 = 0.f;
            }
            arrive_warp(&mrg_empty[0]);
          }
        }
      }
    }
    // the last item's total
    if (MODE == MODE_COLSUM && ok && hc == 0 && items_done > 0) colsum_flush(items_done - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// SpecPC with split segment groups: add each key's per-head partial sums over
// the groups in group order, then take the max over query heads.  One thread
// per key, 256 keys per block (consecutive threads read consecutive floats).
__global__ void __launch_bounds__(256)
    specpc_merge_kernel(const float* __restrict__ part, int n_in, int n_blocks, int groups, int hq,
                        float* __restrict__ scores) {
  const int blk = blockIdx.x;
  const int r = threadIdx.x;
  const int j = (blk % n_blocks) * 256 + r;
  if (j >= n_in) return;
  const float* base = part + static_cast<size_t>(blk) * groups * hq * 256 + r;
  float best = -INFINITY;
  for (int qh = 0; qh < hq; ++qh) {
    float sum = 0.f;
    for (int g = 0; g < groups; ++g) sum += base[(static_cast<size_t>(g) * hq + qh) * 256];
    best = fmaxf(best, sum);
  }
  scores[static_cast<size_t>(blk / n_blocks) * n_in + j] = best;
}

cudaError_t launch_specpc_merge(const float* part, int batch, int n_in, int n_blocks, int groups, int hq,
                                float* scores, cudaStream_t stream) {
  specpc_merge_kernel<<<batch * n_blocks, 256, 0, stream>>>(part, n_in, n_blocks, groups, hq, scores);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// host-side launch helpers
// ---------------------------------------------------------------------------
template <int MODE, int D>
static cudaError_t launch_one(const CUtensorMap& amap, const CUtensorMap& bmap, const ScoreParams& p, int grid,
                              cudaStream_t stream) {
  using C = Cfg<MODE, D>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(score_kernel<MODE, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  score_kernel<MODE, D><<<grid, kThreads, C::kSmemBytes, stream>>>(amap, bmap, p);
  return cudaGetLastError();
}

cudaError_t launch_score(int mode, int head_dim, const CUtensorMap& amap, const CUtensorMap& bmap,
                         const ScoreParams& p, int grid, cudaStream_t stream) {
  if (head_dim == 128) {
    if (mode == MODE_LSE) return launch_one<MODE_LSE, 128>(amap, bmap, p, grid, stream);
    if (mode == MODE_COLSUM) return launch_one<MODE_COLSUM, 128>(amap, bmap, p, grid, stream);
    if (mode == MODE_COLSUM_PC) return launch_one<MODE_COLSUM_PC, 128>(amap, bmap, p, grid, stream);
  } else if (head_dim == 64) {
    if (mode == MODE_LSE) return launch_one<MODE_LSE, 64>(amap, bmap, p, grid, stream);
    if (mode == MODE_COLSUM) return launch_one<MODE_COLSUM, 64>(amap, bmap, p, grid, stream);
    if (mode == MODE_COLSUM_PC) return launch_one<MODE_COLSUM_PC, 64>(amap, bmap, p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

int score_smem_bytes(int mode, int head_dim) {
  if (head_dim == 128) {
    if (mode == MODE_LSE) return Cfg<MODE_LSE, 128>::kSmemBytes;
    if (mode == MODE_COLSUM) return Cfg<MODE_COLSUM, 128>::kSmemBytes;
    if (mode == MODE_COLSUM_PC) return Cfg<MODE_COLSUM_PC, 128>::kSmemBytes;
  } else {
    if (mode == MODE_LSE) return Cfg<MODE_LSE, 64>::kSmemBytes;
    if (mode == MODE_COLSUM) return Cfg<MODE_COLSUM, 64>::kSmemBytes;
    if (mode == MODE_COLSUM_PC) return Cfg<MODE_COLSUM_PC, 64>::kSmemBytes;
  }
  return 0;
}

}  // namespace spk
