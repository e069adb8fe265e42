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
// row, one walk counts their keys above and equal to T, a prefix over warps
// (and CTAs) gives each its output offset and its share of the ties (lowest
// index first), and a second walk writes the indices.  No sort and no list:
// any k, deterministic, ties to the lower index.
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
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
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
// segment [c * seg, (c + 1) * seg).  It stages its scores plus the pooling
// halo in shared memory (cp.async, kDepth tiles in flight), pools them tile
// by tile and overwrites each tile with its keys, so the row is read from
// HBM once and no key goes back to memory.  The three histogram levels and
// the per-CTA counts are summed over distributed shared memory; every CTA
// takes the same decisions from the same sums.

constexpr int kSegCap = 16384;     // keys per CTA at two CTAs per SM
constexpr int kSegMax = 40960;     // keys per CTA at one CTA per SM
constexpr int kClMax = 8;          // portable cluster size
constexpr int kRMax = kTile / 2;   // radius the one-tile look-ahead covers
constexpr int kDepth = 6;          // tiles of scores in flight per CTA
constexpr size_t kClSmemLimit = 227 * 1024;   // dynamic shared memory of one CTA

struct ClShared {
  uint32_t hist[2][kBins];
  int warp_tot[33];
  int warp_gt[kSelWarps], warp_eq[kSelWarps];
  int pub[2];                      // this CTA's keys above T and equal to T
  int s_bin, s_rem;
  int base_pos, base_eq;           // output offset and ties of the CTAs before this one
};

__host__ __device__ constexpr size_t cl_head_bytes() { return (sizeof(ClShared) + 15) / 16 * 16; }

// Shared-memory floats of a segment of seg keys with radius r: whole tiles,
// the halo, and the vector over-read of the last window.
__host__ __device__ constexpr int cl_buf_floats(int seg, int r) {
  return (seg + kTile - 1) / kTile * kTile + 2 * r + 4;
}

// Pooled values of the four consecutive candidates j0 .. j0 + 3 whose
// windows start at w[0] (w = scores[j0 - R] in the staged buffer, padding
// outside the row), from ceil((4 + 2R) / 4) 16-byte loads.
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
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float m = x[e];
#pragma unroll
      for (int t = 1; t <= 2 * R; ++t) m = fmaxf(m, x[e + t]);
      p[e] = m;
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

__device__ __forceinline__ void pool4(const float* w, int r, int mode, int j0, int n, float (&p)[4]) {
  switch (r) {
    case 0: pool4_fixed<0>(w, mode, j0, n, p); break;
    case 1: pool4_fixed<1>(w, mode, j0, n, p); break;
    case 2: pool4_fixed<2>(w, mode, j0, n, p); break;
    case 3: pool4_fixed<3>(w, mode, j0, n, p); break;
    case 4: pool4_fixed<4>(w, mode, j0, n, p); break;
    case 5: pool4_fixed<5>(w, mode, j0, n, p); break;
    case 6: pool4_fixed<6>(w, mode, j0, n, p); break;
    default:
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = pool_staged(w + e, r, mode, j0 + e, n);
  }
}

// find_bin over the cluster's summed histograms hist[h][0, NB): PER = NB /
// kSelThreads consecutive bins per thread (one when NB < kSelThreads), read
// from every CTA of the cluster in rank order.
template <int NB>
__device__ __forceinline__ void find_bin_cluster(ClShared& sh, int h, int remaining, int cl) {
  constexpr int PER = NB >= kSelThreads ? NB / kSelThreads : 1;
  static_assert(PER == 1 || PER == 8, "bins per thread");
  const int top = NB - 1 - static_cast<int>(threadIdx.x) * PER;   // this thread's highest bin
  int cnt[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) cnt[q] = 0;                       // cnt[q]: bin top - PER + 1 + q
  if (top >= 0) {
    const uint32_t a = smem_u32(&sh.hist[h][top - PER + 1]);
    for (int rank = 0; rank < cl; ++rank) {
      const uint32_t ra = dsmem_addr(a, static_cast<uint32_t>(rank));
      if constexpr (PER == 8) {
        const uint4 x = dsmem_ld4(ra), y = dsmem_ld4(ra + 16);
        cnt[0] += x.x; cnt[1] += x.y; cnt[2] += x.z; cnt[3] += x.w;
        cnt[4] += y.x; cnt[5] += y.y; cnt[6] += y.z; cnt[7] += y.w;
      } else {
        cnt[0] += static_cast<int>(dsmem_ld(ra));
      }
    }
  }
  int v = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) v += cnt[q];
  int total;
  const int before = block_exclusive_scan(v, sh.warp_tot, total);   // candidates in higher bins
  if (before < remaining && remaining <= before + v) {
    int cum = before;
#pragma unroll
    for (int q = PER - 1; q >= 0; --q) {
      if (cum + cnt[q] >= remaining) {
        sh.s_bin = top - (PER - 1 - q);
        sh.s_rem = remaining - cum;
        break;
      }
      cum += cnt[q];
    }
  }
  __syncthreads();
}

// Histogram (into hist[h], cleared here) of the segment's keys that match
// `prefix` on their top `known` bits, by their next `width` bits.
__device__ __forceinline__ void segment_hist(ClShared& sh, int h, const uint32_t* keys, int len, uint32_t prefix,
                                             int known, int width) {
  const int nb = 1 << width;
  for (int b = threadIdx.x; b < nb; b += kSelThreads) sh.hist[h][b] = 0;
  __syncthreads();
  const int shift = 32 - known - width;
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  const int nv = (len + 3) / 4;
  for (int vi = threadIdx.x; vi < nv; vi += kSelThreads) {
    const uint4 w = kv[vi];
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (4 * vi + e < len && (k4[e] >> (32 - known)) == prefix) atomicAdd(&sh.hist[h][(k4[e] >> shift) & (nb - 1)], 1u);
  }
}

__global__ void __launch_bounds__(kSelThreads, 2)
    topk_cluster_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int pool_mode, int k, int n_tail,
                        int* __restrict__ idx, float* __restrict__ pooled, int seg) {
  extern __shared__ __align__(16) unsigned char cl_smem[];
  ClShared& sh = *reinterpret_cast<ClShared*>(cl_smem);
  float* sc = reinterpret_cast<float*>(cl_smem + cl_head_bytes());
  uint32_t* keys = reinterpret_cast<uint32_t*>(sc);   // keys overwrite their tile of scores

  const int tid = threadIdx.x;
  const int cl = static_cast<int>(cluster_nctarank());
  const int c = static_cast<int>(cluster_ctarank());
  const int u = blockIdx.x / cl;
  const int n = n_cand, r = pool_r;
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

  const float* s = scores + static_cast<size_t>(u) * n;
  float* pout = pooled ? pooled + static_cast<size_t>(u) * n : nullptr;

  // 1. sc[i] = scores[lo - r + i] for i < len + 2r (padding outside the
  // row), group g = sc[g * kTile, (g + 1) * kTile); pooling tile t needs the
  // groups up to t + 1 (2r <= kTile)
  const float pad = pool_mode == POOL_MAX ? -INFINITY : 0.f;
  const int span = len + 2 * r;
  auto load_group = [&](int g) {
    if (g * kTile < span) {
#pragma unroll
      for (int q = 0; q < kTile / kSelThreads; ++q) {
        const int i = g * kTile + q * kSelThreads + tid;
        const int jj = lo - r + i;
        if (i < span) {
          if (jj >= 0 && jj < n) cp_async4(sc + i, s + jj);
          else sc[i] = pad;
        }
      }
    }
    cp_async_commit();
  };
  if (select)
    for (int b = tid; b < kBins; b += kSelThreads) sh.hist[0][b] = 0;
#pragma unroll 1
  for (int g = 0; g < kDepth; ++g) load_group(g);

  const int nt = (len + kTile - 1) / kTile;
  uint32_t run_bin = kBins, run_cnt = 0;
  uint4 pend = make_uint4(0u, 0u, 0u, 0u);             // keys of the previous tile
#pragma unroll 1
  for (int t = 0; t < nt; ++t) {
    cp_async_wait<kDepth - 2>();                        // this thread's groups <= t + 1
    __syncthreads();                                    // everyone's; tile t - 1 pooled
    const int i0 = t * kTile + 4 * tid;
    if (t > 0 && select) *reinterpret_cast<uint4*>(keys + i0 - kTile) = pend;
    float p[4];
    pool4(sc + i0, r, pool_mode, lo + i0, n, p);
    uint32_t k4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = i0 + e < len;
      k4[e] = valid ? float_key(p[e]) : 0u;
      if (valid && pout) pout[lo + i0 + e] = p[e];
      if (valid && select) {
        const uint32_t bin = k4[e] >> 20;
        if (bin == run_bin) {
          ++run_cnt;
        } else {
          if (run_cnt) atomicAdd(&sh.hist[0][run_bin], run_cnt);
          run_bin = bin;
          run_cnt = 1;
        }
      }
    }
    pend = make_uint4(k4[0], k4[1], k4[2], k4[3]);
    load_group(t + kDepth);
  }
  cp_async_wait<0>();
  if (!select) return;
  if (run_cnt) atomicAdd(&sh.hist[0][run_bin], run_cnt);
  __syncthreads();                                      // every tile pooled
  if (nt > 0) *reinterpret_cast<uint4*>(keys + (nt - 1) * kTile + 4 * tid) = pend;
  cluster_sync();                                       // keys and level-1 histograms complete

  // 2. the exact key T of the C-th largest over the row: 12 + 12 + 8 bits
  find_bin_cluster<kBins>(sh, 0, C, cl);
  uint32_t prefix = static_cast<uint32_t>(sh.s_bin);
  int remaining = sh.s_rem;
  segment_hist(sh, 1, keys, len, prefix, 12, 12);
  cluster_sync();
  find_bin_cluster<kBins>(sh, 1, remaining, cl);
  prefix = (prefix << 12) | static_cast<uint32_t>(sh.s_bin);
  remaining = sh.s_rem;
  segment_hist(sh, 0, keys, len, prefix, 24, 8);      // hist[0] was last read before the previous barrier
  cluster_sync();
  find_bin_cluster<256>(sh, 0, remaining, cl);
  const uint32_t T = (prefix << 8) | static_cast<uint32_t>(sh.s_bin);
  const int take_eq = sh.s_rem;                         // keys equal to T to take, lowest index first

  // 3. ordered emission: warp-contiguous, 128-key-aligned chunks of the
  // segment; counts per warp, then per CTA across the cluster
  const int lane = tid & 31, warp = tid >> 5;
  const int chunk = ((len + kSelWarps - 1) / kSelWarps + 127) & ~127;
  const int beg = min(warp * chunk, len), end = min(beg + chunk, len);
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  int gt = 0, eq = 0;
  for (int j0 = beg; j0 < end; j0 += 128) {
    const int j = j0 + 4 * lane;
    const uint4 w = j < end ? kv[j >> 2] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = j + e < end;
      gt += valid && k4[e] > T;
      eq += valid && k4[e] == T;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    sh.warp_gt[warp] = gt;
    sh.warp_eq[warp] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    int tg = 0, te = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      tg += sh.warp_gt[w];
      te += sh.warp_eq[w];
    }
    sh.pub[0] = tg;
    sh.pub[1] = te;
  }
  cluster_sync();                                       // every CTA's counts published
  if (tid == 0) {
    int pos = 0, eqb = 0;
    const uint32_t a = smem_u32(&sh.pub[0]);
    for (int rank = 0; rank < c; ++rank) {
      const uint32_t ra = dsmem_addr(a, static_cast<uint32_t>(rank));
      const int g2 = static_cast<int>(dsmem_ld(ra)), e2 = static_cast<int>(dsmem_ld(ra + 4));
      pos += g2 + min(max(take_eq - eqb, 0), e2);
      eqb += e2;
    }
    sh.base_pos = pos;
    sh.base_eq = eqb;
  }
  cluster_arrive();                                     // no remote reads past this point
  __syncthreads();
  int pos = sh.base_pos, eq_before = sh.base_eq;
  for (int w = 0; w < warp; ++w) {
    const int we = sh.warp_eq[w];
    pos += sh.warp_gt[w] + min(max(take_eq - eq_before, 0), we);
    eq_before += we;
  }
  const int my_eq = min(max(take_eq - eq_before, 0), eq);   // ties this warp takes
  int eq_seen = 0;
  for (int j0 = beg; j0 < end; j0 += 128) {
    const int j = j0 + 4 * lane;
    const uint4 w = j < end ? kv[j >> 2] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t k4[4] = {w.x, w.y, w.z, w.w};
    int n_eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) n_eq += (j + e < end) && k4[e] == T;
    int eq_pre = n_eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, eq_pre, o);
      if (lane >= o) eq_pre += y;
    }
    int rank = eq_seen + eq_pre - n_eq;
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
      if (sel[e]) out[at++] = lo + j + e;
    pos += __shfl_sync(0xffffffffu, sel_pre, 31);
    eq_seen += __shfl_sync(0xffffffffu, eq_pre, 31);
  }
  cluster_wait();                                       // no CTA leaves while its counts may be read
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
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kClSmemLimit));
    if (e != cudaSuccess) return e;
    configured_device = dev;
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
  e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, n_cand, r, pool_mode, k, n_tail, idx, pooled, plan.seg);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace spk
