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
//      shared memory (five independent loads per thread in flight); every
//      pooled value is formed there and counted in a 4096-bin histogram of
//      its key's top 12 bits.  The bin B1 that holds the C-th largest key
//      follows from one scan of the histogram.
//   2. sweep 2 forms the same pooled values again (the same fp32 operations,
//      so the same keys): keys in bins above B1 are selected outright and
//      their indices collected; keys in B1 are collected with their index as
//      candidates.  Both lists live in shared memory.
//   3. the candidates are sorted by (key descending, index ascending), the
//      first C - |selected| of them complete the selection, and the C indices
//      are sorted ascending: ties go to the lower index, the output is
//      ordered, and the result does not depend on the order in which threads
//      appended to the lists.
// When C exceeds 2048, or more than 2048 candidates share bin B1 (long runs of
// equal values), a general path takes over: the keys go to the workspace and
// a three-level radix select (12 + 12 + 8 bits) finds the exact C-th key T;
// an ordered ballot walk over each warp's contiguous share of the row emits
// the indices ascending, keys equal to T lowest index first.
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
constexpr int kListMax = 2048;              // shared-memory selection lists

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

// Ascending bitonic sort of a[0, P) in shared memory, P a power of two.
template <typename T>
__device__ __forceinline__ void bitonic_sort(T* a, int P) {
  for (int k = 2; k <= P; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < P; i += kSelThreads) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const T x = a[i], y = a[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

struct SelShared {
  float tile[kTile + 2 * kHaloMax];
  uint32_t hist[kBins];
  unsigned long long cand[kListMax];   // (~key << 32) | index: ascending = key desc, index asc
  int list[kListMax];
  int warp_tot[33];
  int s_bin, s_rem, n_a, n_b;
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

// Warp-aggregated append of the lanes with pred to a shared list: returns
// the lane's slot (or -1), one atomic per warp.
__device__ __forceinline__ int warp_append(int* counter, bool pred) {
  const uint32_t m = __ballot_sync(0xffffffffu, pred);
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == 0 && m) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xffffffffu, base, 0);
  return pred ? base + __popc(m & ((1u << lane) - 1u)) : -1;
}

// General path (C > kListMax, or more than kListMax keys share even a 24-bit
// prefix with the C-th largest): three radix levels over the keys in the
// workspace, then an ordered ballot emission.
__device__ __noinline__ void select_general(SelShared& sh, int n, int C, const uint32_t* __restrict__ keys,
                                            int* __restrict__ out) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  uint32_t* hist = sh.hist;
  __syncthreads();
  for (int b = tid; b < kBins; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  key_sweep(keys, n, [&](int, bool valid, uint32_t key) { hist_add(hist, valid ? key >> 20 : kBins); });
  __syncthreads();
  find_bin(hist, kBins, C, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  uint32_t prefix = static_cast<uint32_t>(sh.s_bin);        // top 12 bits of T
  int remaining = sh.s_rem;
  for (int b = tid; b < kBins; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  key_sweep(keys, n, [&](int, bool valid, uint32_t key) {
    hist_add(hist, valid && (key >> 20) == prefix ? (key >> 8) & 4095u : kBins);
  });
  __syncthreads();
  find_bin(hist, kBins, remaining, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  prefix = (prefix << 12) | static_cast<uint32_t>(sh.s_bin);   // top 24 bits of T
  remaining = sh.s_rem;
  for (int b = tid; b < 256; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  key_sweep(keys, n, [&](int, bool valid, uint32_t key) {
    hist_add(hist, valid && (key >> 8) == prefix ? key & 255u : kBins);
  });
  __syncthreads();
  find_bin(hist, 256, remaining, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  const uint32_t T = (prefix << 8) | static_cast<uint32_t>(sh.s_bin);
  const int take_eq = sh.s_rem;   // keys equal to T to take, lowest index first

  // ordered emission: warp w owns [w * chunk, (w + 1) * chunk)
  const int chunk = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
  const int beg = warp * chunk < n ? warp * chunk : n;
  const int end = beg + chunk < n ? beg + chunk : n;
  int gt = 0, eq = 0;
  for (int j0 = beg; j0 < end; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < end ? keys[j] : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, j < end && key > T));
    eq += __popc(__ballot_sync(0xffffffffu, j < end && key == T));
  }
  int total;
  // one value per warp: lane 0 carries it, the others add nothing
  const int eq_before = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? eq : 0, sh.warp_tot, total), 0);
  int my_eq = take_eq - eq_before;
  my_eq = my_eq < 0 ? 0 : (my_eq > eq ? eq : my_eq);
  int pos = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? gt + my_eq : 0, sh.warp_tot, total), 0);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int j0 = beg; j0 < end; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < end ? keys[j] : 0u;
    const bool is_eq = j < end && key == T;
    const uint32_t eq_bal = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = (j < end && key > T) || (is_eq && static_cast<int>(__popc(eq_bal & lt_mask)) < my_eq);
    const uint32_t sel_bal = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(sel_bal & lt_mask)] = j;
    pos += __popc(sel_bal);
    my_eq -= __popc(eq_bal);
  }
}

// The candidates (sh.n_b <= kListMax of them) sorted by (key desc, index
// asc) complete the selected list with `need` entries; the C indices are
// then sorted ascending and written.
__device__ __forceinline__ void finish_selection(SelShared& sh, int need, int C, int* __restrict__ out) {
  const int tid = threadIdx.x;
  const int n_a = sh.n_a, n_b = sh.n_b;
  const int pb = pow2_at_least(n_b);
  for (int t = n_b + tid; t < pb; t += kSelThreads) sh.cand[t] = ~0ull;
  __syncthreads();
  bitonic_sort(sh.cand, pb);
  for (int t = tid; t < need; t += kSelThreads) sh.list[n_a + t] = static_cast<int>(sh.cand[t] & 0xffffffffu);
  const int pc = pow2_at_least(C);
  for (int t = C + tid; t < pc; t += kSelThreads) sh.list[t] = 0x7fffffff;
  __syncthreads();
  bitonic_sort(sh.list, pc);
  for (int t = tid; t < C; t += kSelThreads) out[t] = sh.list[t];
}

__global__ void __launch_bounds__(kSelThreads, 4)
    topk_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int pool_mode, int k, int n_tail,
                int* __restrict__ idx, float* __restrict__ pooled, uint32_t* __restrict__ keys_ws, int key_stride) {
  extern __shared__ __align__(16) uint8_t sel_smem[];   // 50 KB: above the 48 KB of static shared memory
  SelShared& sh = *reinterpret_cast<SelShared*>(sel_smem);
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

  // 1. pooled values -> (optional output), keys to the workspace, histogram of their top 12 bits
  for (int b = tid; b < kBins; b += kSelThreads) sh.hist[b] = 0;
  if (tid == 0) { sh.n_a = 0; sh.n_b = 0; }
  __syncthreads();
  // Histogram adds are run-length aggregated per thread: the pooled values
  // crowd into a few bins, and contended shared-memory atomics on the same
  // bin serialize, so a thread adds a bin's count once per run of equal bins.
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
  if (C > kListMax) {
    select_general(sh, n, C, keys, out);
    return;
  }
  find_bin(sh.hist, kBins, C, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  const uint32_t b1 = static_cast<uint32_t>(sh.s_bin);
  const int need1 = sh.s_rem;    // keys of bin b1 still to take (>= 1)
  for (int b = tid; b < kBins; b += kSelThreads) sh.hist[b] = 0;
  __syncthreads();

  // 2. bins above b1 are selected; bin b1's keys are candidates, histogrammed on their next 12 bits
  key_sweep(keys, n, [&](int j, bool valid, uint32_t key) {
    const uint32_t bin = key >> 20;
    const bool in_b = valid && bin == b1;
    if (in_b) atomicAdd(&sh.hist[(key >> 8) & 4095u], 1u);
    const int pa = warp_append(&sh.n_a, valid && bin > b1);   // fewer than C <= kListMax of these
    if (pa >= 0) sh.list[pa] = j;
    const int pb = warp_append(&sh.n_b, in_b);
    if (pb >= 0 && pb < kListMax) sh.cand[pb] = (static_cast<unsigned long long>(~key) << 32) | static_cast<uint32_t>(j);
  });
  __syncthreads();
  if (sh.n_b <= kListMax) {
    finish_selection(sh, need1, C, out);
    return;
  }

  // 3. too many candidates: refine bin b1 by the next 12 bits
  find_bin(sh.hist, kBins, need1, sh.warp_tot, &sh.s_bin, &sh.s_rem);
  const uint32_t p24 = (b1 << 12) | static_cast<uint32_t>(sh.s_bin);
  const int need2 = sh.s_rem;
  if (tid == 0) sh.n_b = 0;
  __syncthreads();
  key_sweep(keys, n, [&](int j, bool valid, uint32_t key) {
    const uint32_t pre = key >> 8;
    const int pa = warp_append(&sh.n_a, valid && (key >> 20) == b1 && pre > p24);
    if (pa >= 0) sh.list[pa] = j;
    const int pb = warp_append(&sh.n_b, valid && pre == p24);
    if (pb >= 0 && pb < kListMax) sh.cand[pb] = (static_cast<unsigned long long>(~key) << 32) | static_cast<uint32_t>(j);
  });
  __syncthreads();
  if (sh.n_b <= kListMax) {
    finish_selection(sh, need2, C, out);
    return;
  }
  select_general(sh, n, C, keys, out);   // long runs of equal values
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
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(SelShared)));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  topk_kernel<<<units, kSelThreads, sizeof(SelShared), stream>>>(scores, n_cand, pool_kernel / 2, pool_mode, k, n_tail, idx,
                                                 pooled, static_cast<uint32_t*>(ws), key_stride(n_cand));
  return cudaGetLastError();
}

}  // namespace spk
