// select.cu -- local pooling and deterministic top-k selection with a kept tail.
//
// "Draft-based Approximate Inference for LLMs" (paper notes): section 关键设计
// keeps the top-C_max KV pairs plus the window; section 损失函数 / 训练策略
// smooths SpecPC scores with local pooling so that kept tokens form runs.
// The pages name local pooling without its kind: max pooling (the workloads'
// "pool 7") and average pooling (mean over the clipped window) are offered.
//
// Pooled values are turned into order-preserving 32-bit keys (a larger float
// gives a larger key); the C-th largest key T is found exactly by three
// histogram levels (the top 12 bits, then the next 12, then the last 8, each
// later level counting only the keys that match the prefix found so far),
// and the selection {key > T} u {the first take_eq keys == T} is emitted in
// ascending index order: warps own contiguous, 128-key-aligned shares of the
// row and count their keys above and equal to T (one walk, or the last
// histogram level's sweep in the cluster kernel), a prefix over warps (and
// CTAs) gives each its output offset and its share of the ties (lowest index
// first), and a walk writes the indices.  No sort and no list: any k,
// deterministic, ties to the lower index.
//
// Two kernels do this.  topk_cluster_kernel (rows up to 8 x kSegMax
// candidates, pooling radius up to kTile / 2) splits a row over a cluster of
// up to eight CTAs that keep their segment's scores, then keys, in shared
// memory and sum their histograms and counts over distributed shared memory:
// the row is read from HBM once.  topk_kernel (one CTA per row, any length)
// stages tiles of 2048 scores plus the halo, writes the keys to a workspace
// (rows padded to 16 bytes) and sweeps them there with 16-byte loads.
#include "common.cuh"
#include "score.cuh"

namespace spk {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 4096;
constexpr int kTile = 2048;                 // candidates per staged tile
constexpr int kHaloMax = 256;               // pooling radius served from the staged tile
constexpr int kTileLoads = (kTile + 2 * kHaloMax + kSelThreads - 1) / kSelThreads;   // 5

// Monotone map from finite floats to uint32 (larger float -> larger key);
// -0 is folded onto +0 so that the two compare equal, as they do as floats.
// No float maps to 0.
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
  const uint32_t k = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return k + (k == 0u);   // 0 is kept free (it marks an empty position); only the all-ones NaN moves
}

// Exclusive prefix sum over the CTA (kSelThreads threads); also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kSelWarps ? warp_tot[lane] : 0;
    int wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    if (lane < kSelWarps) warp_tot[lane] = wx - w;   // exclusive warp offsets
    if (lane == 31) warp_tot[32] = wx;
  }
  __syncthreads();
  const int out = warp_tot[warp] + x - v;
  total = warp_tot[32];
  __syncthreads();
  return out;
}

// Given the histogram of the candidates that still match the prefix, find
// the bin holding the remaining-th largest: bins are scanned from the top,
// nbins / kSelThreads consecutive bins per thread.  Returns the bin (in
// s_bin) and the count still to take inside it (in s_rem).
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, int remaining, int* warp_tot,
                                         int* s_bin, int* s_rem) {
  const int per = nbins / kSelThreads > 0 ? nbins / kSelThreads : 1;
  const int top = nbins - 1 - threadIdx.x * per;   // this thread's highest bin
  int v = 0;
  for (int i = 0; i < per; ++i)
    if (top - i >= 0) v += static_cast<int>(hist[top - i]);
  int total;
  const int before = block_exclusive_scan(v, warp_tot, total);   // candidates in higher bins
  if (before < remaining && remaining <= before + v) {
    int cum = before;
    for (int i = 0; i < per; ++i) {
      const int h = static_cast<int>(hist[top - i]);
      if (cum + h >= remaining) {
        *s_bin = top - i;
        *s_rem = remaining - cum;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
}

// Pooled value of candidate j.  `w` points at scores[j - r] inside a staged
// tile whose slots outside [0, n) hold the padding (-inf for max, 0 for the
// average), so the window needs no bounds tests.  The average divides the
// sum of the clipped window (in window order) by its length.
__device__ __forceinline__ float pool_staged(const float* w, int r, int mode, int j, int n) {
  if (mode == POOL_MAX) {
    float m = -INFINITY;
    for (int t = 0; t <= 2 * r; ++t) m = fmaxf(m, w[t]);
    return m;
  }
  float s = 0.f;
  for (int t = 0; t <= 2 * r; ++t) s += w[t];
  const int lo = j - r < 0 ? 0 : j - r;
  const int hi = j + r > n - 1 ? n - 1 : j + r;
  return __fdiv_rn(s, static_cast<float>(hi - lo + 1));
}

// The same value read straight from global memory (radii beyond the halo).
__device__ __forceinline__ float pool_direct(const float* s, int r, int mode, int j, int n) {
  const int lo = j - r < 0 ? 0 : j - r;
  const int hi = j + r > n - 1 ? n - 1 : j + r;
  if (mode == POOL_MAX) {
    float m = -INFINITY;
    for (int t = lo; t <= hi; ++t) m = fmaxf(m, s[t]);
    return m;
  }
  float acc = 0.f;
  for (int t = lo; t <= hi; ++t) acc += s[t];
  return __fdiv_rn(acc, static_cast<float>(hi - lo + 1));
}

// Calls f(j, valid, pooled_j) for every candidate j of the row, warp-uniformly
// (every lane of every warp calls f the same number of times; lanes past the
// end pass valid = false), tile by tile.
template <typename F>
__device__ __forceinline__ void pooled_sweep(const float* __restrict__ s, int n, int r, int mode, float* tile,
                                             F&& f) {
  const int tid = threadIdx.x;
  const bool staged = r <= kHaloMax;
  const float pad = mode == POOL_MAX ? -INFINITY : 0.f;
  const int len = kTile + 2 * r;
  // scores[base - r, base + kTile + r) with padding outside [0, n); the next
  // tile's loads are issued before this tile is pooled, so their latency
  // overlaps the pooling
  float v[kTileLoads];
  auto load_tile = [&](int base) {
#pragma unroll
    for (int q = 0; q < kTileLoads; ++q) {
      const int t = tid + q * kSelThreads;
      const int jj = base - r + t;
      v[q] = (t < len && jj >= 0 && jj < n) ? __ldg(s + jj) : pad;
    }
  };
  if (staged) load_tile(0);
  for (int base = 0; base < n; base += kTile) {
    if (staged) {
#pragma unroll
      for (int q = 0; q < kTileLoads; ++q) {
        const int t = tid + q * kSelThreads;
        if (t < len) tile[t] = v[q];
      }
      __syncthreads();
      if (base + kTile < n) load_tile(base + kTile);
    }
#pragma unroll 1
    for (int i = 0; i < kTile / kSelThreads; ++i) {
      const int off = i * kSelThreads + tid;
      const int j = base + off;
      const bool valid = j < n;
      float p = 0.f;
      if (valid) p = staged ? pool_staged(tile + off, r, mode, j, n) : pool_direct(s, r, mode, j, n);
      f(j, valid, p);
    }
    if (staged) __syncthreads();
  }
}

struct SelShared {
  float tile[kTile + 2 * kHaloMax];
  uint32_t hist[kBins];
  int warp_tot[33];
  int s_bin, s_rem;
};

// Calls f(j, valid, key_j) for every key of the row (keys padded to a
// multiple of 4 per row, 16-byte aligned), warp-uniformly: each thread loads
// four 16-byte vectors per round before using any of them.
template <typename F>
__device__ __forceinline__ void key_sweep(const uint32_t* __restrict__ keys, int n, F&& f) {
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  const int nv = (n + 3) / 4;
  for (int base = 0; base < nv; base += 4 * kSelThreads) {
    uint4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int vi = base + q * kSelThreads + threadIdx.x;
      w[q] = vi < nv ? kv[vi] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = 4 * (base + q * kSelThreads + threadIdx.x);
      f(j + 0, j + 0 < n, w[q].x);
      f(j + 1, j + 1 < n, w[q].y);
      f(j + 2, j + 2 < n, w[q].z);
      f(j + 3, j + 3 < n, w[q].w);
    }
  }
}

// Histogram of the keys that match `prefix` on their top `known` bits, by
// their next `width` bits (plain atomics: these keys spread over the bins).
__device__ __forceinline__ void prefix_hist(SelShared& sh, const uint32_t* __restrict__ keys, int n, uint32_t prefix,
                                            int known, int width) {
  const int nb = 1 << width;
  for (int b = threadIdx.x; b < nb; b += kSelThreads) sh.hist[b] = 0;
  __syncthreads();
  const int shift = 32 - known - width;
  key_sweep(keys, n, [&](int, bool valid, uint32_t key) {
    if (valid && (key >> (32 - known)) == prefix) atomicAdd(&sh.hist[(key >> shift) & (nb - 1)], 1u);
  });
  __syncthreads();
}

// Ordered emission of the selection {key > T} u {the first take_eq keys ==
// T}: warp w owns a contiguous, 128-key-aligned share of the row; one walk
// counts its keys above and equal to T, a CTA-wide prefix gives every warp
// its output offset and its share of the ties, and a second walk writes the
// indices in ascending order (lane l holds keys 4l .. 4l + 3 of each
// 128-key step; output positions by warp scans).
__device__ __forceinline__ void emit_ordered(SelShared& sh, const uint32_t* __restrict__ keys, int n, uint32_t T,
                                             int take_eq, int* __restrict__ out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = ((n + kSelWarps - 1) / kSelWarps + 127) & ~127;
  const int beg = min(warp * chunk, n), end = min(beg + chunk, n);
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  int gt = 0, eq = 0;
  for (int j0 = beg; j0 < end; j0 += 4 * 128) {
    uint4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q * 128 + 4 * lane;
      w[q] = j < end ? kv[j >> 2] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q * 128 + 4 * lane;
      const uint32_t k4[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool valid = j + e < end;
        gt += valid && k4[e] > T;
        eq += valid && k4[e] == T;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  int total;
  // one value per warp: lane 0 carries it, the others add nothing
  const int eq_before = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? eq : 0, sh.warp_tot, total), 0);
  const int my_eq = min(max(take_eq - eq_before, 0), eq);   // ties this warp takes, lowest index first
  int pos = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? gt + my_eq : 0, sh.warp_tot, total), 0);
  int eq_seen = 0;
  for (int j0 = beg; j0 < end; j0 += 128) {
    const int j = j0 + 4 * lane;
    const uint4 w = j < end ? kv[j >> 2] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
    int n_eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) n_eq += (j + e < end) && k4[e] == T;
    int eq_pre = n_eq;                                 // inclusive warp scan of the ties
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, eq_pre, o);
      if (lane >= o) eq_pre += y;
    }
    int rank = eq_seen + eq_pre - n_eq;                // ties before this lane's first
    bool sel[4];
    int n_sel = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = j + e < end;
      const bool is_eq = valid && k4[e] == T;
      sel[e] = (valid && k4[e] > T) || (is_eq && rank < my_eq);
      rank += is_eq;
      n_sel += sel[e];
    }
    int sel_pre = n_sel;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sel_pre, o);
      if (lane >= o) sel_pre += y;
    }
    int at = pos + sel_pre - n_sel;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (sel[e]) out[at++] = j + e;
    pos += __shfl_sync(0xffffffffu, sel_pre, 31);
    eq_seen += __shfl_sync(0xffffffffu, eq_pre, 31);
  }
}

__global__ void __launch_bounds__(kSelThreads, 4)
    topk_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int pool_mode, int k, int n_tail,
                int* __restrict__ idx, float* __restrict__ pooled, uint32_t* __restrict__ keys_ws, int key_stride) {
  __shared__ SelShared sh;
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  const int n = n_cand;
  const int C = k < n ? k : n;
  const size_t out_len = static_cast<size_t>(C) + n_tail;
  int* out = idx + static_cast<size_t>(u) * out_len;

  // kept tail (the window)
  for (int t = tid; t < n_tail; t += kSelThreads) out[C + t] = n + t;
  if (C == 0 && pooled == nullptr) return;

  const float* s = scores + static_cast<size_t>(u) * n;
  uint32_t* keys = keys_ws + static_cast<size_t>(u) * key_stride;
  float* pout = pooled ? pooled + static_cast<size_t>(u) * n : nullptr;
  const bool select = C > 0 && C < n;

  // 1. pooled values -> (optional output), keys to the workspace, histogram
  // of their top 12 bits.  The adds are run-length aggregated per thread: the
  // pooled values crowd into a few bins, and contended shared-memory atomics
  // on one bin serialize.
  for (int b = tid; b < kBins; b += kSelThreads) sh.hist[b] = 0;
  __syncthreads();
  uint32_t run_bin = kBins, run_cnt = 0;
  pooled_sweep(s, n, pool_r, pool_mode, sh.tile, [&](int j, bool valid, float p) {
    if (!valid) return;
    if (pout) pout[j] = p;
    if (!select) return;
    const uint32_t key = float_key(p);
    keys[j] = key;
    const uint32_t bin = key >> 20;
    if (bin == run_bin) {
      ++run_cnt;
    } else {
      if (run_cnt) atomicAdd(&sh.hist[run_bin], run_cnt);
      run_bin = bin;
      run_cnt = 1;
    }
  });
  if (run_cnt) atomicAdd(&sh.hist[run_bin], run_cnt);
  if (C == 0) return;
  if (C >= n) {
    for (int j = tid; j < n; j += kSelThreads) out[j] = j;
    return;
  }
  __syncthreads();               // keys and histogram complete

  // 2. the exact key T of the C-th largest: 12 + 12 + 8 bits, the later
  // levels histogramming only the keys that match the prefix so far
  find_bin(sh.hist, kBins, C, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  uint32_t prefix = static_cast<uint32_t>(sh.s_bin);
  int remaining = sh.s_rem;
  prefix_hist(sh, keys, n, prefix, 12, 12);
  find_bin(sh.hist, kBins, remaining, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  prefix = (prefix << 12) | static_cast<uint32_t>(sh.s_bin);
  remaining = sh.s_rem;
  prefix_hist(sh, keys, n, prefix, 24, 8);
  find_bin(sh.hist, 256, remaining, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  const uint32_t T = (prefix << 8) | static_cast<uint32_t>(sh.s_bin);
  const int take_eq = sh.s_rem;  // keys equal to T to take, lowest index first

  // 3. ordered emission
  emit_ordered(sh, keys, n, T, take_eq, out);
}

// ---------------------------------------------------------------------------
// Cluster path.  The row's candidates are split over a cluster of CL CTAs
// (CL in {1, 2, 4, 8}, the smallest whose share fits): CTA c owns the
// segment [c * seg, (c + 1) * seg).  It copies its scores plus the pooling
// halo into shared memory (16-byte cp.async, every round in flight at
// once), pools them round by round and overwrites each pooled round with its
// keys, so the row is read from HBM once and no key goes back to memory.
//
// Layout: the buffer starts at the 16-byte boundary at or below the global
// position of scores[lo - r]; with a = that position mod 4, buffer slot m
// (four floats) holds the pooling windows' starts of candidates
// 4m - a .. 4m - a + 3, whose keys later replace those four floats.  Slots
// stay aligned in both memories whatever n, lo and r are.
//
// Exchanges between the cluster's CTAs (after a cluster barrier, over
// distributed shared memory, always summed in rank order so that every CTA
// takes the same decisions):
//   level 1 and 2 (4096 bins): 64-bin super-bin sums, then the 64 bins of
//     the chosen super-bin (one remote load per thread and step);
//   level 3 (256 bins): the bins themselves, which also give every CTA's
//     count of keys above and equal to T (with the count above the 24-bit
//     prefix that each CTA publishes), so that the output offsets need no
//     further barrier.
// Per-warp counts for the ordered emission come from the level-3 sweep (keys
// above the 24-bit prefix, and keys on it); only a warp holding keys on the
// prefix walks its share again.

constexpr int kSegCap = 16384;     // keys per CTA at two CTAs per SM
constexpr int kSegMax = 40960;     // keys per CTA at one CTA per SM
constexpr int kClMax = 8;          // portable cluster size
constexpr int kRMax = kTile / 2;   // radius whose window the next load round covers
constexpr int kRound = kSelThreads;              // slots (four candidates) per round
constexpr int kSuperBins = 64;                   // bins per super-bin (4096-bin levels)
constexpr int kSupers = kBins / kSuperBins;      // 64
constexpr size_t kClSmemLimit = 227 * 1024;      // dynamic shared memory of one CTA

struct ClShared {
  uint32_t hist[2][kBins];         // this CTA's level histograms
  uint32_t super[2][kSupers];      // super-bin sums of levels 1 and 2
  uint32_t tot_super[kSupers];     // cluster sums (local scratch)
  uint32_t tot_bin[kSupers];
  uint32_t tot3[256];
  int warp_tot[33];
  int warp_above[kSelWarps], warp_on[kSelWarps];   // level-3 sweep: above / on the 24-bit prefix
  int warp_gt[kSelWarps], warp_eq[kSelWarps];
  int rank_gt[kClMax], rank_eq[kClMax];
  int above24;                     // this CTA's keys above the 24-bit prefix (published)
  int s_bin, s_rem;
  int base_pos, base_eq;           // output offset and ties of the CTAs before this one
};

__host__ __device__ constexpr size_t cl_head_bytes() { return (sizeof(ClShared) + 15) / 16 * 16; }

// Shared-memory floats of a segment of seg keys with radius r: the slots of
// the copied range (up to three floats of alignment, the halo) and the
// vector over-read of the last windows.
__host__ __device__ constexpr int cl_buf_floats(int seg, int r) {
  return (seg + 2 * r + 3 + 3) / 4 * 4 + 32;
}

// Pooled values of the four consecutive candidates j0 .. j0 + 3 whose
// windows start at w[0] .. w[3] (16-byte aligned), from ceil((4 + 2R) / 4)
// 16-byte loads.  Padding in the buffer stands for positions outside the row.
template <int R>
__device__ __forceinline__ void pool4_fixed(const float* w, int mode, int j0, int n, float (&p)[4]) {
  constexpr int NV = (4 + 2 * R + 3) / 4;
  float x[4 * NV];
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const float4 v = reinterpret_cast<const float4*>(w)[q];
    x[4 * q + 0] = v.x;
    x[4 * q + 1] = v.y;
    x[4 * q + 2] = v.z;
    x[4 * q + 3] = v.w;
  }
  if (mode == POOL_MAX) {
    if constexpr (2 * R >= 3) {
      // out_e = max x[e .. e + 2R]: all four share x[3 .. 2R]; the rest is
      // a suffix of x[0 .. 2] on the left and a prefix of x[2R + 1 ..] on
      // the right (max is exact, so the grouping does not change a value)
      float core = x[3];
#pragma unroll
      for (int t = 4; t <= 2 * R; ++t) core = fmaxf(core, x[t]);
      const float l1 = fmaxf(x[1], x[2]), l0 = fmaxf(x[0], l1);
      const float r1 = x[2 * R + 1], r2 = fmaxf(r1, x[2 * R + 2]), r3 = fmaxf(r2, x[2 * R + 3]);
      p[0] = fmaxf(core, l0);
      p[1] = max3f(core, l1, r1);
      p[2] = max3f(core, x[2], r2);
      p[3] = fmaxf(core, r3);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float m = x[e];
#pragma unroll
        for (int t = 1; t <= 2 * R; ++t) m = fmaxf(m, x[e + t]);
        p[e] = m;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float s = 0.f;
#pragma unroll
      for (int t = 0; t <= 2 * R; ++t) s += x[e + t];
      const int j = j0 + e;
      const int lo = j - R < 0 ? 0 : j - R;
      const int hi = j + R > n - 1 ? n - 1 : j + R;
      p[e] = __fdiv_rn(s, static_cast<float>(hi - lo + 1));
    }
  }
}

// Wait until at most `pending` (clamped to 7) of this thread's cp.async
// groups are still in flight; waiting for more than needed is harmless.
__device__ __forceinline__ void cp_async_wait_upto(int pending) {
  switch (pending < 7 ? (pending < 0 ? 0 : pending) : 7) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

// 64-bin super-bin sums of hist[h] into super[h]: eight bins per thread,
// eight threads per super-bin.
__device__ __forceinline__ void super_sums(ClShared& sh, int h) {
  const uint4* hv = reinterpret_cast<const uint4*>(sh.hist[h]) + 2 * threadIdx.x;
  const uint4 x = hv[0], y = hv[1];
  uint32_t v = x.x + x.y + x.z + x.w + y.x + y.y + y.z + y.w;
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  if ((threadIdx.x & 7) == 0) sh.super[h][threadIdx.x >> 3] = v;
}

// Within warp 0: the entry holding the remaining-th largest of cnt[0, 64)
// (scanned from the top, two entries per lane).  Lane 0 returns it in
// (*bin, *rem); every lane returns the same.
__device__ __forceinline__ void warp_find64(const uint32_t* cnt, int remaining, int* bin, int* rem) {
  const int lane = threadIdx.x & 31;
  const int hi = 63 - 2 * lane;                 // this lane's entries: hi, hi - 1
  const int c0 = static_cast<int>(cnt[hi]), c1 = static_cast<int>(cnt[hi - 1]);
  int x = c0 + c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const int before = x - c0 - c1;               // in higher entries
  const bool mine = before < remaining && remaining <= x;
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int src = who ? __ffs(who) - 1 : 0;
  const int b = remaining <= before + c0 ? hi : hi - 1;
  const int rr = remaining <= before + c0 ? remaining - before : remaining - before - c0;
  *bin = __shfl_sync(0xffffffffu, b, src);
  *rem = __shfl_sync(0xffffffffu, rr, src);
}

// Level exchange over 4096 bins: the super-bin holding the remaining-th
// largest key over the cluster, then the bin inside it.  Result in
// sh.s_bin / sh.s_rem.  Called after a cluster barrier that published
// super[h] and hist[h] of every CTA.
__device__ __forceinline__ void find_bin_4096(ClShared& sh, int h, int remaining, int cl) {
  const int t = threadIdx.x;
  if (t < kSupers) {
    sh.tot_super[t] = 0;
    sh.tot_bin[t] = 0;
  }
  __syncthreads();
  if (t < cl * kSupers) {
    const uint32_t v = dsmem_ld(dsmem_addr(smem_u32(&sh.super[h][t % kSupers]), t / kSupers));
    if (v) atomicAdd(&sh.tot_super[t % kSupers], v);
  }
  __syncthreads();
  if (t < 32) {
    int sb, rem;
    warp_find64(sh.tot_super, remaining, &sb, &rem);
    if (t == 0) {
      sh.s_bin = sb;
      sh.s_rem = rem;
    }
  }
  __syncthreads();
  const int sb = sh.s_bin, rem = sh.s_rem;
  if (t < cl * kSupers) {
    const uint32_t v = dsmem_ld(dsmem_addr(smem_u32(&sh.hist[h][sb * kSuperBins + t % kSupers]), t / kSupers));
    if (v) atomicAdd(&sh.tot_bin[t % kSupers], v);
  }
  __syncthreads();
  if (t < 32) {
    int b, r2;
    warp_find64(sh.tot_bin, rem, &b, &r2);
    if (t == 0) {
      sh.s_bin = sb * kSuperBins + b;
      sh.s_rem = r2;
    }
  }
  __syncthreads();
}

// Level exchange over the 256 bins of level 3 (hist[0][0, 256)), which also
// fills rank_gt / rank_eq: every CTA's keys on the 24-bit prefix above and
// at the chosen bin.  Result in sh.s_bin / sh.s_rem.
__device__ __forceinline__ void find_bin_256(ClShared& sh, int remaining, int cl) {
  const int t = threadIdx.x, b = t & 255, g = t >> 8;     // g: 0 or 1
  sh.tot3[b] = 0;                                           // both halves write the same zero
  if (t < kClMax) {
    sh.rank_gt[t] = 0;
    sh.rank_eq[t] = 0;
  }
  __syncthreads();
  uint32_t v[kClMax / 2];
#pragma unroll
  for (int q = 0; q < kClMax / 2; ++q) {
    const int rank = g + 2 * q;
    v[q] = rank < cl ? dsmem_ld(dsmem_addr(smem_u32(&sh.hist[0][b]), rank)) : 0u;
  }
  uint32_t s = 0;
#pragma unroll
  for (int q = 0; q < kClMax / 2; ++q) s += v[q];
  if (s) atomicAdd(&sh.tot3[b], s);
  __syncthreads();
  // warp 0: eight bins per lane, scanned from the top
  if (t < 32) {
    const int lane = t;
    uint32_t c[8];
    int x = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = sh.tot3[255 - 8 * lane - q];
      x += static_cast<int>(c[q]);
    }
    const int own = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int before = x - own;
    if (before < remaining && remaining <= x) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int cq = static_cast<int>(c[q]);
        if (before + cq >= remaining) {
          sh.s_bin = 255 - 8 * lane - q;
          sh.s_rem = remaining - before;
          break;
        }
        before += cq;
      }
    }
  }
  __syncthreads();
  const int B3 = sh.s_bin;
#pragma unroll
  for (int q = 0; q < kClMax / 2; ++q) {
    const int rank = g + 2 * q;
    if (rank < cl) {
      // a warp's 32 bins are one rank's: reduce, one add per warp
      uint32_t above = b > B3 ? v[q] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      if ((t & 31) == 0 && above) atomicAdd(&sh.rank_gt[rank], static_cast<int>(above));
      if (b == B3) sh.rank_eq[rank] = static_cast<int>(v[q]);
    }
  }
  __syncthreads();
}

// Level-1 histogram (top 12 key bits) of the segment's keys.  Thread t takes
// the eight consecutive slots 8t .. 8t + 7 of each 4096-slot block (32
// consecutive candidates), visiting them rotated by its lane so that the
// eight lanes of each quarter-warp read different 16-byte columns (no bank
// conflict); equal bins are counted in runs.  Empty positions (key 0) are
// counted in bin 0 and taken out by the caller.
__device__ __forceinline__ void level1_hist(ClShared& sh, const uint32_t* keys, int n_groups) {
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  const int lane = threadIdx.x & 31;
  uint32_t run_bin = kBins, run_cnt = 0;
  auto add = [&](uint32_t bin, uint32_t cnt) {
    if (bin == run_bin) {
      run_cnt += cnt;
    } else {
      if (run_cnt) atomicAdd(&sh.hist[0][run_bin], run_cnt);
      run_bin = bin;
      run_cnt = cnt;
    }
  };
  for (int base = 8 * static_cast<int>(threadIdx.x); base < n_groups; base += 8 * kSelThreads) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int m = base + ((q + lane) & 7);
      if (m >= n_groups) continue;
      const uint4 w = kv[m];
      if (((w.x ^ w.y) | (w.x ^ w.z) | (w.x ^ w.w)) < (1u << 20)) {
        add(w.x >> 20, 4u);                                       // one bin for the four
      } else {
        add(w.x >> 20, 1u);
        add(w.y >> 20, 1u);
        add(w.z >> 20, 1u);
        add(w.w >> 20, 1u);
      }
    }
  }
  if (run_cnt) atomicAdd(&sh.hist[0][run_bin], run_cnt);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// R >= 0: the pooling radius, unrolled; R < 0: any radius up to kRMax (pool_r).
template <int R>
__global__ void __launch_bounds__(kSelThreads, 2)
    topk_cluster_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int pool_mode, int k, int n_tail,
                        int* __restrict__ idx, float* __restrict__ pooled, int seg, int vec_ok) {
  extern __shared__ __align__(16) unsigned char cl_smem[];
  ClShared& sh = *reinterpret_cast<ClShared*>(cl_smem);
  float* buf = reinterpret_cast<float*>(cl_smem + cl_head_bytes());
  uint32_t* keys = reinterpret_cast<uint32_t*>(buf);   // keys replace their slot's scores

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cl = static_cast<int>(cluster_nctarank());
  const int c = static_cast<int>(cluster_ctarank());
  const int u = blockIdx.x / cl;
  const int n = n_cand, r = R >= 0 ? R : pool_r;
  const int C = k < n ? k : n;
  const size_t out_len = static_cast<size_t>(C) + n_tail;
  int* out = idx + static_cast<size_t>(u) * out_len;
  const int lo = c * seg;
  const int len = max(0, min(seg, n - lo));          // candidates of this CTA

  if (c == 0)
    for (int t = tid; t < n_tail; t += kSelThreads) out[C + t] = n + t;
  if (C == 0 && pooled == nullptr) return;
  const bool select = C > 0 && C < n;
  if (C >= n && C > 0)
    for (int j = tid; j < len; j += kSelThreads) out[lo + j] = lo + j;
  if (!select && pooled == nullptr) return;

  float* pout = pooled ? pooled + static_cast<size_t>(u) * n : nullptr;

  // 1. copies: slot m <- global floats [g0 + 4m, g0 + 4m + 4), g0 the
  // 16-byte boundary at or below row position lo - r; positions outside the
  // row hold the padding.  One commit group per round of kRound slots.
  const float* s = scores + static_cast<size_t>(u) * n;          // the row
  const long long want = static_cast<long long>(u) * n + lo - r;  // global position of window start 0
  const int a = static_cast<int>(want & 3);
  const int j0 = lo - r - a;                                      // row position of slot 0's first float
  const int n_slots = len > 0 ? (a + len + 2 * r + 3) / 4 : 0;
  const int n_groups = len > 0 ? (a + len + 3) / 4 : 0;           // slots whose candidates include one < len
  const int load_rounds = (n_slots + kRound - 1) / kRound;
  const int pool_rounds = (n_groups + kRound - 1) / kRound;
  const float pad = pool_mode == POOL_MAX ? -INFINITY : 0.f;
  if (select) {
    for (int b = tid; b < kBins; b += kSelThreads) {
      sh.hist[0][b] = 0;
      sh.hist[1][b] = 0;
    }
  }
#pragma unroll 1
  for (int lr = 0; lr < load_rounds; ++lr) {
    const int m = lr * kRound + tid;
    if (m < n_slots) {
      const int jr = j0 + 4 * m;                                  // row position of the slot's first float
      float* dst = buf + 4 * m;
      if (vec_ok && jr >= 0 && jr + 3 < n) {
        cp_async16(dst, s + jr);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (jr + e >= 0 && jr + e < n) cp_async4(dst + e, s + jr + e);
          else dst[e] = pad;
        }
      }
    }
    cp_async_commit();
  }

  // 2. pool round by round; round t's windows reach into load round t + 1.
  // The keys of round t - 1 are stored once every thread has pooled it.
  uint4 pend = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
  for (int t = 0; t < pool_rounds; ++t) {
    cp_async_wait_upto(load_rounds - (t + 2));
    __syncthreads();
    const int m = t * kRound + tid;
    if (t > 0 && select) *reinterpret_cast<uint4*>(keys + 4 * (m - kRound)) = pend;   // a full round
    if (m < n_groups) {
      const int i0 = 4 * m - a;                                   // candidate of the slot's first float
      float p[4];
      if constexpr (R >= 0) {
        pool4_fixed<R>(buf + 4 * m, pool_mode, lo + i0, n, p);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = pool_staged(buf + 4 * m + e, r, pool_mode, lo + i0 + e, n);
      }
      uint32_t k4[4];
      bool v4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v4[e] = i0 + e >= 0 && i0 + e < len;
        k4[e] = v4[e] ? float_key(p[e]) : 0u;
        if (v4[e] && pout) pout[lo + i0 + e] = p[e];
      }
      pend = make_uint4(k4[0], k4[1], k4[2], k4[3]);
    } else {
      pend = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_wait<0>();
  if (!select) return;
  __syncthreads();                                                // every round pooled
  if (pool_rounds > 0) {
    const int m = (pool_rounds - 1) * kRound + tid;
    if (m < n_groups) *reinterpret_cast<uint4*>(keys + 4 * m) = pend;
  }
  __syncthreads();                                                // every key stored
  // slots [0, n_groups) hold 4 * n_groups - len empty positions (key 0):
  // a before candidate 0, the rest after candidate len - 1
  const int n_empty = 4 * n_groups - len;
  level1_hist(sh, keys, n_groups);
  __syncthreads();
  if (tid == 0 && n_empty > 0) sh.hist[0][0] -= n_empty;          // the empty positions' bin
  __syncthreads();
  super_sums(sh, 0);
  cluster_sync();                                                 // S1: level 1 of every CTA

  // 3. the exact key T of the C-th largest over the row: 12 + 12 + 8 bits
  find_bin_4096(sh, 0, C, cl);
  const uint32_t B1 = static_cast<uint32_t>(sh.s_bin);
  int remaining = sh.s_rem;
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  for (int m = tid; m < n_groups; m += kSelThreads) {
    const uint4 w = kv[m];
    const uint32_t mx = max(max(w.x, w.y), max(w.z, w.w)), mn = min(min(w.x, w.y), min(w.z, w.w));
    if ((mx >> 20) < B1 || (mn >> 20) > B1) continue;             // no key of the slot in bin B1
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if ((k4[e] >> 20) == B1) atomicAdd(&sh.hist[1][(k4[e] >> 8) & 0xfffu], 1u);
  }
  __syncthreads();
  if (tid == 0 && B1 == 0 && n_empty > 0) sh.hist[1][0] -= n_empty;
  __syncthreads();
  super_sums(sh, 1);
  cluster_sync();                                                 // S2: level 2 of every CTA
  find_bin_4096(sh, 1, remaining, cl);
  const uint32_t P24 = (B1 << 12) | static_cast<uint32_t>(sh.s_bin);
  remaining = sh.s_rem;

  // level 3 over warp-contiguous shares of the slots (the emission's
  // partition): keys above the 24-bit prefix and on it, per warp
  for (int b = tid; b < 256; b += kSelThreads) sh.hist[0][b] = 0;   // read remotely only before S2
  __syncthreads();
  const int chunk = ((n_groups + kSelWarps - 1) / kSelWarps + 31) & ~31;   // slots, whole 32-slot steps
  const int beg = min(warp * chunk, n_groups), end = min(beg + chunk, n_groups);
  int above = 0, on = 0;
  for (int m0 = beg; m0 < end; m0 += 32) {
    const int m = m0 + lane;
    if (m < end) {
      const uint4 w = kv[m];
      const uint32_t mx = max(max(w.x, w.y), max(w.z, w.w));
      if ((mx >> 8) >= P24) {                                     // else every key is below the prefix
        const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t top = k4[e] >> 8;
          above += top > P24;
          if (top == P24) {
            ++on;
            atomicAdd(&sh.hist[0][k4[e] & 0xffu], 1u);
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    above += __shfl_xor_sync(0xffffffffu, above, o);
    on += __shfl_xor_sync(0xffffffffu, on, o);
  }
  if (lane == 0) {
    sh.warp_above[warp] = above;
    sh.warp_on[warp] = on;
  }
  __syncthreads();
  if (tid == 0) {
    int s2 = 0;
    for (int w = 0; w < kSelWarps; ++w) s2 += sh.warp_above[w];
    sh.above24 = s2;
    if (P24 == 0 && n_empty > 0) sh.hist[0][0] -= n_empty;        // empty positions sit on prefix 0
  }
  cluster_sync();                                                 // S3: level 3 and above24 of every CTA
  find_bin_256(sh, remaining, cl);
  const uint32_t B3 = static_cast<uint32_t>(sh.s_bin);
  const uint32_t T = (P24 << 8) | B3;
  const int take_eq = sh.s_rem;                                   // keys equal to T to take, lowest index first
  if (tid == 0) {
    // keys above T and equal to T in the CTAs before this one
    int pos = 0, eqb = 0;
    for (int rank = 0; rank < c; ++rank) {
      const int g2 = static_cast<int>(dsmem_ld(dsmem_addr(smem_u32(&sh.above24), rank))) + sh.rank_gt[rank];
      const int e2 = sh.rank_eq[rank];
      pos += g2 + min(max(take_eq - eqb, 0), e2);
      eqb += e2;
    }
    sh.base_pos = pos;
    sh.base_eq = eqb;
  }
  cluster_arrive();                                               // no remote reads past this point

  // per-warp counts: exact from level 3 unless the warp holds keys on the prefix
  int gt = sh.warp_above[warp], eq = 0;
  if (sh.warp_on[warp] > 0) {
    int g2 = 0;
    for (int m0 = beg; m0 < end; m0 += 32) {
      const int m = m0 + lane;
      if (m < end) {
        const uint4 w = kv[m];
        const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
        const int i0 = 4 * m - a;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (i0 + e < 0 || i0 + e >= len || (k4[e] >> 8) != P24) continue;
          g2 += (k4[e] & 0xffu) > B3;
          eq += (k4[e] & 0xffu) == B3;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g2 += __shfl_xor_sync(0xffffffffu, g2, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    gt += g2;
  }
  if (lane == 0) {
    sh.warp_gt[warp] = gt;
    sh.warp_eq[warp] = eq;
  }
  __syncthreads();
  int pos = sh.base_pos, eq_before = sh.base_eq;
  for (int w = 0; w < warp; ++w) {
    const int we = sh.warp_eq[w];
    pos += sh.warp_gt[w] + min(max(take_eq - eq_before, 0), we);
    eq_before += we;
  }
  const int my_eq = min(max(take_eq - eq_before, 0), eq);        // ties this warp takes
  const bool partial = my_eq > 0 && my_eq < eq;                  // only then do tie ranks matter

  // 4. ordered emission over the warp's share, 128 keys per step
  const uint32_t lt = lanemask_lt();
  int eq_seen = 0;
  for (int m0 = beg; m0 < end; m0 += 32) {
    const int m = m0 + lane;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (m < end) w = kv[m];
    const uint32_t mx = max(max(w.x, w.y), max(w.z, w.w));
    if (__ballot_sync(0xffffffffu, mx >= T) == 0) continue;       // no key of the step at or above T
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
    const int i0 = 4 * m - a;
    uint32_t gt4 = 0, eq4 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gt4 |= static_cast<uint32_t>(k4[e] > T) << e;               // empty positions hold 0 < T
      eq4 |= static_cast<uint32_t>(k4[e] == T) << e;
    }
    uint32_t sel4;
    if (!partial) {
      sel4 = gt4 | (my_eq > 0 ? eq4 : 0u);
    } else {
      const int n_eq = __popc(eq4);
      int eq_pre = n_eq;                                          // inclusive warp scan of the ties
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, eq_pre, o);
        if (lane >= o) eq_pre += y;
      }
      int rank = eq_seen + eq_pre - n_eq;
      sel4 = gt4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((eq4 >> e) & 1u) {
          if (rank < my_eq) sel4 |= 1u << e;
          ++rank;
        }
      }
      eq_seen += __shfl_sync(0xffffffffu, eq_pre, 31);
    }
    // exclusive prefix of the per-lane counts (0..4) from three ballots
    const int ns = __popc(sel4);
    const uint32_t q0 = __ballot_sync(0xffffffffu, ns & 1), q1 = __ballot_sync(0xffffffffu, ns & 2),
                   q2 = __ballot_sync(0xffffffffu, ns & 4);
    int at = pos + __popc(q0 & lt) + 2 * __popc(q1 & lt) + 4 * __popc(q2 & lt);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if ((sel4 >> e) & 1u) out[at++] = lo + i0 + e;
    pos += __popc(q0) + 2 * __popc(q1) + 4 * __popc(q2);
  }
  cluster_wait();                                                 // no CTA leaves while it may be read
}

}  // namespace

// Keys of one row, padded to a multiple of four (16-byte vectors).
static int key_stride(int n_cand) { return n_cand > 0 ? (n_cand + 3) & ~3 : 0; }

size_t topk_ws_bytes(int units, int n_cand) {
  return static_cast<size_t>(units) * static_cast<size_t>(key_stride(n_cand)) * sizeof(uint32_t);
}

// Cluster shape of a row: the smallest power-of-two cluster whose share of
// the row fits kSegCap keys (two CTAs per SM), else eight CTAs with up to
// kSegMax keys each (one CTA per SM); cl = 0 selects the workspace kernel
// (longer rows, or pooling radii beyond one tile's look-ahead).
struct ClusterPlan {
  int cl = 0, seg = 0;
  size_t smem = 0;
};

static ClusterPlan cluster_plan(int n_cand, int r) {
  ClusterPlan p;
  if (n_cand <= 0 || r > kRMax) return p;
  for (int c = 1; c <= kClMax; c *= 2) {
    const int seg = key_stride((n_cand + c - 1) / c);
    if (seg <= kSegCap || (c == kClMax && seg <= kSegMax)) {
      p.cl = c;
      p.seg = seg;
      p.smem = cl_head_bytes() + static_cast<size_t>(cl_buf_floats(seg, r)) * sizeof(float);
      break;
    }
  }
  if (p.smem > kClSmemLimit) p.cl = 0;
  return p;
}

template <int R>
static cudaError_t launch_cluster(cudaLaunchConfig_t& cfg, const float* scores, int n_cand, int r, int pool_mode,
                                  int k, int n_tail, int* idx, float* pooled, int seg, int vec_ok) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(topk_cluster_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kClSmemLimit));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<R>, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, seg,
                         vec_ok);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                        int n_tail, int* idx, float* pooled, void* ws, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  const int r = pool_kernel / 2;
  const ClusterPlan plan = cluster_plan(n_cand, r);
  if (plan.cl == 0) {
    topk_kernel<<<units, kSelThreads, 0, stream>>>(scores, n_cand, r, pool_mode, k, n_tail, idx, pooled,
                                                   static_cast<uint32_t*>(ws), key_stride(n_cand));
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units) * static_cast<unsigned>(plan.cl));
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(plan.cl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int vec_ok = (reinterpret_cast<uintptr_t>(scores) & 15u) == 0;
  switch (r) {
    case 0: return launch_cluster<0>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 1: return launch_cluster<1>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 2: return launch_cluster<2>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 3: return launch_cluster<3>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 4: return launch_cluster<4>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 5: return launch_cluster<5>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    case 6: return launch_cluster<6>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
    default: return launch_cluster<-1>(cfg, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg, vec_ok);
  }
}

}  // namespace spk
