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
//   warp 8   : TMA producer (A tiles once per segment, B tiles streamed)
//   warp 9   : TMEM allocator + single-thread UMMA issuer (128 x N x 16 bf16)
//   warps 0-7: epilogue; warpgroup t owns A tile t, each thread one TMEM lane.
// TMEM holds 2 accumulator stages x 2 A tiles x 128 fp32 columns (512 cols).
// No atomics: every output element is reduced by exactly one thread in a
// fixed order, so results are bitwise reproducible.
#include "common.cuh"
#include "score.cuh"

namespace spk {

__device__ int g_device_error = 0;
__device__ int g_device_error_site = 0;

namespace {

constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;

template <int MODE, int D>
struct Cfg {
  static constexpr int kTileBytes = 128 * D * 2;          // 128 rows x D bf16
  static constexpr int kAtoms = D / 64;                    // 128-byte swizzle atoms along K
  static constexpr int kAStages = (MODE == MODE_LSE) ? 1 : 2;
  static constexpr int kBStages = (MODE == MODE_LSE) ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 4);
  static constexpr int kABytes = 2 * kTileBytes;
  static constexpr int kSmemA = kAStages * kABytes;
  static constexpr int kSmemB = kBStages * kTileBytes;
  static constexpr int kLseFloats = (MODE == MODE_LSE) ? 0 : 2 * kRowsMax;
  static constexpr int kAccFloats = (MODE == MODE_COLSUM_PC) ? kGroupMax * 256 : 0;
  static constexpr int kSmemBytes = 1024 + kSmemA + kSmemB + 4 * (kLseFloats + kAccFloats);
};

// Error sites: mode * 100 + role * 10 + barrier.
__device__ __forceinline__ int site(int mode, int role, int which) { return mode * 100 + role * 10 + which; }

__device__ __forceinline__ int n_segments(const ScoreParams& p, int mode) {
  return mode == MODE_COLSUM_PC ? p.hkv * p.layers_used : 1;
}

// (item, segment) -> unit, its 3-D tensor coordinate, first A row.
__device__ __forceinline__ void decode(const ScoreParams& p, int mode, int item, int seg, int& u, int& tc,
                                       int& a_row0) {
  if (mode == MODE_COLSUM_PC) {
    const int b = item / p.n_blocks;
    const int h = seg / p.layers_used, lu = seg % p.layers_used;
    u = (b * p.layers_used + lu) * p.hkv + h;
    a_row0 = (item % p.n_blocks) * 256;
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
// pass-1 epilogue: online log2-sum-exp2 over 32 keys of one row
// ---------------------------------------------------------------------------
__device__ __forceinline__ void lse_update(const uint32_t (&v)[32], int jb, int c, float c2, float& m,
                                           float& l) {
  if (jb >= c) return;
  float x[32];
  if (jb + 32 <= c) {
#pragma unroll
    for (int k = 0; k < 32; ++k) x[k] = __uint_as_float(v[k]);
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) x[k] = (jb + k < c) ? __uint_as_float(v[k]) : -INFINITY;
  }
  float mx = x[0];
#pragma unroll
  for (int k = 1; k < 32; ++k) mx = fmaxf(mx, x[k]);
  const float mn = fmaxf(m, mx * c2);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    s0 += ex2_approx(fmaf(x[k + 0], c2, -mn));
    s1 += ex2_approx(fmaf(x[k + 1], c2, -mn));
    s2 += ex2_approx(fmaf(x[k + 2], c2, -mn));
    s3 += ex2_approx(fmaf(x[k + 3], c2, -mn));
  }
  l = fmaf(l, ex2_approx(m - mn), (s0 + s1) + (s2 + s3));
  m = mn;
}

// ---------------------------------------------------------------------------
// pass-2 epilogue: sum over 32 query rows nb..nb+31 of 2^(c2 x - off[row])
// ---------------------------------------------------------------------------
__device__ __forceinline__ float colsum32(const uint32_t (&v)[32], const float* off, int nb, float c2) {
  const float4* o4 = reinterpret_cast<const float4*>(off + nb);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 o = o4[k / 4];
    s0 += ex2_approx(fmaf(__uint_as_float(v[k + 0]), c2, -o.x));
    s1 += ex2_approx(fmaf(__uint_as_float(v[k + 1]), c2, -o.y));
    s2 += ex2_approx(fmaf(__uint_as_float(v[k + 2]), c2, -o.z));
    s3 += ex2_approx(fmaf(__uint_as_float(v[k + 3]), c2, -o.w));
  }
  return (s0 + s1) + (s2 + s3);
}

// Same, for a key j that some rows cannot see: row n (head-local i = n % R)
// sees key j only if j < c0 + i.
__device__ __forceinline__ float colsum32_masked(const uint32_t (&v)[32], const float* off, int nb, float c2,
                                                 int j, int c0, int R) {
  float s = 0.f;
  int i = nb % R;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    if (j < c0 + i) s += ex2_approx(fmaf(__uint_as_float(v[k]), c2, -off[nb + k]));
    if (++i == R) i = 0;
  }
  return s;
}

}  // namespace

template <int MODE, int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                 const ScoreParams p) {
  using C = Cfg<MODE, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const A_s = smem;
  uint8_t* const B_s = smem + C::kSmemA;
  float* const lse_s = reinterpret_cast<float*>(B_s + C::kSmemB);
  float* const acc_s = lse_s + C::kLseFloats;

  __shared__ __align__(8) uint64_t a_full[2], a_empty[2], b_full[8], b_empty[8], acc_full[2], acc_empty[2],
      off_ready[2], done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  __shared__ float wsum_s[kThreads / 32];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kAStages; ++s) { mbar_init(&a_full[s], 1); mbar_init(&a_empty[s], 1); }
    for (int s = 0; s < C::kBStages; ++s) { mbar_init(&b_full[s], 1); mbar_init(&b_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 8); }
    for (int s = 0; s < 2; ++s) mbar_init(&off_ready[s], kEpiThreads);
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_map(&amap);
    tma_prefetch_map(&bmap);
  }
  if (MODE == MODE_COLSUM_PC && threadIdx.x < kEpiThreads)
    for (int n = threadIdx.x; n < C::kAccFloats; n += kEpiThreads) acc_s[n] = 0.f;
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
  const int nseg = n_segments(p, MODE);
  const int nb = b_tiles(p, MODE);

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t a_stage = 0, a_phase = 0, b_stage = 0, b_phase = 0;
      int a_last[2] = {-1, -1};
      int b_last[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        for (int seg = 0; ok && seg < nseg; ++seg) {
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
            mbar_arrive_expect_tx(&b_full[b_stage], C::kTileBytes);
            uint8_t* bdst = B_s + b_stage * C::kTileBytes;
#pragma unroll
            for (int a = 0; a < C::kAtoms; ++a)
              tma_load_3d(bdst + a * 16384, &bmap, &b_full[b_stage], a * 64, bt * 128, tc);
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
          if (a_last[s] >= 0) mbar_wait(&a_full[s], a_last[s], &never, site(MODE, 0, 8), 100000000ull);
        for (int s = 0; s < C::kBStages; ++s)
          if (b_last[s] >= 0) mbar_wait(&b_full[s], b_last[s], &never, site(MODE, 0, 9), 100000000ull);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      uint32_t a_stage = 0, a_phase = 0, b_stage = 0, b_phase = 0, acc_stage = 0, acc_phase = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        for (int seg = 0; ok && seg < nseg; ++seg) {
          int u, tc, a_row0;
          decode(p, MODE, item, seg, u, tc, a_row0);
          const bool act0 = a_tile_active(p, MODE, a_row0, 0);
          const bool act1 = a_tile_active(p, MODE, a_row0, 1);
          if (!(ok = mbar_wait(&a_full[a_stage], a_phase, abort_v, site(MODE, 1, 0)))) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(A_s + a_stage * C::kABytes);
          for (int bt = 0; bt < nb; ++bt) {
            if (!(ok = mbar_wait(&b_full[b_stage], b_phase, abort_v, site(MODE, 1, 1)))) break;
            if (!(ok = mbar_wait(&acc_empty[acc_stage], acc_phase ^ 1, abort_v, site(MODE, 1, 2)))) break;
            tc_fence_after();
            const int n = (MODE == MODE_LSE) ? 128 : chunk_cols(p, bt);
            const uint32_t idesc = idesc_bf16_f32(128, n);
            const uint32_t b_base = smem_u32(B_s + b_stage * C::kTileBytes);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!(t == 0 ? act0 : act1)) continue;
              const uint32_t d_tmem = tmem_base + (acc_stage * 2 + t) * 128;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                umma_bf16_ss(d_tmem, sw128_kmajor_desc(a_base + t * C::kTileBytes + koff),
                             sw128_kmajor_desc(b_base + koff), idesc, kk > 0 ? 1u : 0u);
              }
            }
            umma_commit(&acc_full[acc_stage]);
            umma_commit(&b_empty[b_stage]);
            if (++b_stage == C::kBStages) { b_stage = 0; b_phase ^= 1; }
            if (++acc_stage == 2) { acc_stage = 0; acc_phase ^= 1; }
          }
          if (!ok) break;
          umma_commit(&a_empty[a_stage]);
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
    const int t = warp >> 2;             // A tile (warpgroup)
    const int q = warp & 3;              // TMEM lane quadrant
    const int r = t * 128 + q * 32 + lane;   // A row within the item
    const int etid = threadIdx.x;        // 0..255
    uint32_t acc_stage = 0, acc_phase = 0;
    int seg_count = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      float best = -INFINITY;            // SpecPC: running max over query heads
      float acc = 0.f;                   // SpecKV: column sum of this key
      for (int seg = 0; ok && seg < nseg; ++seg, ++seg_count) {
        int u, tc, a_row0;
        decode(p, MODE, item, seg, u, tc, a_row0);
        const bool active = a_tile_active(p, MODE, a_row0, t);
        if (MODE == MODE_LSE) {
          const int row = a_row0 + r;
          const bool row_ok = active && row < p.rows;
          const int i = row_ok ? row % p.R : 0;
          const int c = min(p.n_in, p.c0 + i);
          float m = -INFINITY, l = 0.f;
          for (int bt = 0; bt < nb; ++bt) {
            ok = mbar_wait(&acc_full[acc_stage], acc_phase, abort_v, site(MODE, 2, 0));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if (active) {
              const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (acc_stage * 2 + t) * 128;
              uint32_t va[32], vb[32];
              tmem_ld32(taddr, va);
              tmem_ld32(taddr + 32, vb);
              tmem_ld_wait2(va, vb);
              const int j0 = bt * 128;
              if (row_ok) {
                lse_update(va, j0, c, p.c2, m, l);
                lse_update(vb, j0 + 32, c, p.c2, m, l);
              }
              __syncwarp();
              tmem_ld32(taddr + 64, va);
              tmem_ld32(taddr + 96, vb);
              tmem_ld_wait2(va, vb);
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[acc_stage]);
              if (row_ok) {
                lse_update(va, j0 + 64, c, p.c2, m, l);
                lse_update(vb, j0 + 96, c, p.c2, m, l);
              }
            } else {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[acc_stage]);
            }
            if (++acc_stage == 2) { acc_stage = 0; acc_phase ^= 1; }
          }
          if (ok && row_ok) {
            float out = m + lg2_approx(l);
            if (p.row_weights != nullptr) out += log2_norm - log2f(p.row_weights[i]);
            p.lse2[static_cast<size_t>(u) * p.rows + row] = out;
          }
        } else {
          // Load this unit's row offsets (lse2, +inf past the last row) into
          // buffer seg_count & 1.  Every epilogue thread arrives on
          // off_ready[buf] after writing; the bounded wait replaces a named
          // barrier so that an aborting warp cannot strand the others.  A
          // buffer is rewritten two segments later, after every thread has
          // passed the wait of the segment in between.
          const int buf = seg_count & 1;
          float* off = lse_s + buf * kRowsMax;
          const int rows_pad = nb * 128;
          const float* src = p.lse2 + static_cast<size_t>(u) * p.rows;
          for (int n = etid; n < rows_pad; n += kEpiThreads) off[n] = (n < p.rows) ? src[n] : INFINITY;
          mbar_arrive(&off_ready[buf]);
          ok = mbar_wait(&off_ready[buf], (seg_count >> 1) & 1, abort_v, site(MODE, 2, 2));
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const int j = a_row0 + r;              // this thread's key
          const bool masked_key = j >= p.c0;     // some rows cannot see it
          float seg_sum = 0.f;
          int cur_head = -1;
          for (int bt = 0; bt < nb; ++bt) {
            ok = mbar_wait(&acc_full[acc_stage], acc_phase, abort_v, site(MODE, 2, 1));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if (active) {
              const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (acc_stage * 2 + t) * 128;
              const int ncols = chunk_cols(p, bt);
              for (int g = 0; g < ncols; g += 32) {
                uint32_t v[32];
                __syncwarp();
                tmem_ld32(taddr + g, v);
                tmem_ld_wait(v);
                const int nb0 = bt * 128 + g;
                if (MODE == MODE_COLSUM) {
                  acc += masked_key ? colsum32_masked(v, off, nb0, p.c2, j, p.c0, p.R) : colsum32(v, off, nb0, p.c2);
                } else {
                  // SpecPC: rows of one query head are contiguous (R = W rows);
                  // rows >= p.rows are padding and belong to no head
                  const int gh = p.rows / p.R;
                  const int h0 = nb0 / p.R, h1 = (nb0 + 31) / p.R;
                  if (h0 >= gh) {
                    // whole group is padding
                  } else if (h0 == h1) {
                    if (h0 != cur_head) {
                      if (cur_head >= 0) acc_s[cur_head * 256 + r] += seg_sum;
                      cur_head = h0;
                      seg_sum = 0.f;
                    }
                    seg_sum += masked_key ? colsum32_masked(v, off, nb0, p.c2, j, p.c0, p.R)
                                          : colsum32(v, off, nb0, p.c2);
                  } else {
                    // a 32-row group that straddles two query heads
                    int i = nb0 % p.R;
                    for (int k = 0; k < 32; ++k) {
                      const int n = nb0 + k;
                      if (n >= p.rows) break;
                      const int hh = n / p.R;
                      if (hh != cur_head) {
                        if (cur_head >= 0) acc_s[cur_head * 256 + r] += seg_sum;
                        cur_head = hh;
                        seg_sum = 0.f;
                      }
                      if (!masked_key || j < p.c0 + i)
                        seg_sum += ex2_approx(fmaf(__uint_as_float(v[k]), p.c2, -off[n]));
                      if (++i == p.R) i = 0;
                    }
                  }
                }
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc_stage]);
            if (++acc_stage == 2) { acc_stage = 0; acc_phase ^= 1; }
          }
          if (MODE == MODE_COLSUM_PC && ok && active) {
            if (cur_head >= 0) acc_s[cur_head * 256 + r] += seg_sum;
            // after the last layer of this KV head: max over its query heads
            const int lu = seg % p.layers_used;
            if (lu == p.layers_used - 1) {
              const int g = p.rows / p.R;
              for (int hh = 0; hh < g; ++hh) {
                best = fmaxf(best, acc_s[hh * 256 + r]);
                acc_s[hh * 256 + r] = 0.f;
              }
            }
          }
        }
      }
      if (!ok) break;
      if (MODE == MODE_COLSUM) {
        int u, tc, a_row0;
        decode(p, MODE, item, 0, u, tc, a_row0);
        const int j = a_row0 + r;
        if (a_tile_active(p, MODE, a_row0, t)) {
          if (j < p.n_pre) p.out0[static_cast<size_t>(u) * p.n_pre + j] = acc;
          else if (j < p.n_cols && p.out1 != nullptr)
            p.out1[static_cast<size_t>(u) * (p.n_in - p.n_pre) + (j - p.n_pre)] = acc;
        }
      } else if (MODE == MODE_COLSUM_PC) {
        const int b = item / p.n_blocks;
        const int j = (item % p.n_blocks) * 256 + r;
        if (j < p.n_cols) p.out0[static_cast<size_t>(b) * p.n_in + j] = best;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
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
  } else {
    if (mode == MODE_LSE) return Cfg<MODE_LSE, 64>::kSmemBytes;
    if (mode == MODE_COLSUM) return Cfg<MODE_COLSUM, 64>::kSmemBytes;
    if (mode == MODE_COLSUM_PC) return Cfg<MODE_COLSUM_PC, 64>::kSmemBytes;
  }
  return 0;
}

}  // namespace spk
