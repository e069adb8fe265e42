// select.cu -- local pooling and deterministic top-k selection with a kept tail.
//
// "Draft-based Approximate Inference for LLMs" (paper notes): section 关键设计
// keeps the top-C_max KV pairs plus the window; section 损失函数 / 训练策略
// smooths SpecPC scores with local pooling so that kept tokens form runs.
// The pages name local pooling without its kind: max pooling (the workloads'
// "pool 7") and average pooling (mean over the clipped window) are offered.
//
// One CTA (512 threads) per row of candidates.  Pooled values are turned into
// order-preserving 32-bit keys (a larger float gives a larger key).
//   1. sweep 1: tiles of 2048 scores plus the pooling halo are staged in
//      shared memory (five independent loads per thread, the next tile's
//      issued before the current one is pooled); every pooled value is
//      formed there, its key written to the workspace (rows padded to 16
//      bytes) and its top 12 bits counted in a 4096-bin histogram
//      (run-length aggregated per thread: the values crowd into few bins).
//   2. the exact key T of the C-th largest, and how many keys equal to T to
//      take, from two more histograms (the next 12, then the last 8 bits) of
//      only the keys that match the prefix found so far; the workspace keys
//      are swept with 16-byte loads, four in flight per thread.
//   3. ordered emission: each warp owns a contiguous share of the row; one
//      walk counts its keys above and equal to T, a CTA prefix gives every
//      warp its output offset and its share of the ties (lowest index
//      first), a second walk writes the indices in ascending order.
// No sort and no shared-memory list: any k, deterministic, ties to the
// lower index.
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

// Add one to hist[bin] for every lane with bin < kBins.  Scores cluster, so
// whole warps often share a bin: the lanes that match lane 0's bin add
// together (one atomic), the others add their own.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
  const uint32_t b0 = __shfl_sync(0xffffffffu, bin, 0);
  const uint32_t same = __ballot_sync(0xffffffffu, bin == b0);
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    if (b0 < kBins) atomicAdd(&hist[b0], __popc(same));
  } else if (bin != b0 && bin < kBins) {
    atomicAdd(&hist[bin], 1u);
  }
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

}  // namespace

// Keys of one row, padded to a multiple of four (16-byte vectors).
static int key_stride(int n_cand) { return n_cand > 0 ? (n_cand + 3) & ~3 : 0; }

size_t topk_ws_bytes(int units, int n_cand) {
  return static_cast<size_t>(units) * static_cast<size_t>(key_stride(n_cand)) * sizeof(uint32_t);
}

cudaError_t launch_topk(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                        int n_tail, int* idx, float* pooled, void* ws, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  topk_kernel<<<units, kSelThreads, 0, stream>>>(scores, n_cand, pool_kernel / 2, pool_mode, k, n_tail, idx,
                                                 pooled, static_cast<uint32_t*>(ws), key_stride(n_cand));
  return cudaGetLastError();
}

}  // namespace spk
