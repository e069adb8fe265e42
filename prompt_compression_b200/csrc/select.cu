// select.cu -- max-pooling and deterministic top-k selection with a kept tail.
//
// "Draft-based Approximate Inference for LLMs" (paper notes): section 关键设计
// keeps the top-C_max KV pairs plus the window; section 损失函数 / 训练策略
// smooths SpecPC scores with local pooling so that kept tokens form runs.
//
// One CTA (512 threads) per row of candidates:
//   1. pooled[j] = max of scores over the clipped window [j-r, j+r]: tiles of
//      scores with their halo are staged in shared memory (coalesced loads);
//      the pooled values are stored as order-preserving 32-bit keys, and a
//      4096-bin histogram of their top 12 bits is built on the way.
//   2. radix select in three passes (12, 12 and 8 bits, most significant
//      first) finds the exact key T of the C-th largest value and how many
//      keys equal to T must be taken; histogram updates are warp-aggregated.
//   3. emission: each warp owns a contiguous run of indices and walks it 32
//      at a time with ballots; one prefix over the warps' counts (keys equal
//      to T, then selected keys) gives every warp its output offset, so the
//      indices come out ascending with ties resolved lowest index first.
#include "common.cuh"
#include "score.cuh"

namespace spk {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 4096;
constexpr int kHaloMax = kSelThreads;   // pooling radius staged through shared memory

// Monotone map from finite floats to uint32 (larger float -> larger key);
// -0 is folded onto +0 so that the two compare equal, as they do as floats.
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Add one to hist[bin] for every lane with bin < kBins, one atomic per
// distinct bin in the warp.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
  const uint32_t peers = __match_any_sync(0xffffffffu, bin);
  if (bin < kBins && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
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
// kBins / kSelThreads consecutive bins per thread.  Returns the bin (in
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

__global__ void __launch_bounds__(kSelThreads, 4)
    topk_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int k, int n_tail, int* __restrict__ idx,
                float* __restrict__ pooled, uint32_t* __restrict__ keys_ws) {
  __shared__ uint32_t hist[kBins];
  __shared__ float tile[kSelThreads + 2 * kHaloMax];
  __shared__ int warp_tot[33];
  __shared__ int s_bin, s_rem;

  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n = n_cand;
  const int C = k < n ? k : n;
  const size_t out_len = static_cast<size_t>(C) + n_tail;
  int* out = idx + static_cast<size_t>(u) * out_len;

  // kept tail (the window)
  for (int t = tid; t < n_tail; t += kSelThreads) out[C + t] = n + t;
  if (C == 0 && pooled == nullptr) return;

  const float* s = scores + static_cast<size_t>(u) * n;
  uint32_t* keys = keys_ws + static_cast<size_t>(u) * n;
  float* pout = pooled ? pooled + static_cast<size_t>(u) * n : nullptr;

  // 1. pooling -> keys, histogram of the top 12 bits
  for (int b = tid; b < kBins; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  const bool staged = pool_r <= kHaloMax;
  for (int base = 0; base < n; base += kSelThreads) {
    const int j = base + tid;
    float m = -INFINITY;
    if (staged) {
      // scores[base - r, base + kSelThreads + r) with -inf outside [0, n):
      // the max over the padded window equals the max over the clipped one
      for (int t = tid; t < kSelThreads + 2 * pool_r; t += kSelThreads) {
        const int jj = base - pool_r + t;
        tile[t] = (jj >= 0 && jj < n) ? s[jj] : -INFINITY;
      }
      __syncthreads();
      if (j < n)
        for (int t = 0; t <= 2 * pool_r; ++t) m = fmaxf(m, tile[tid + t]);
      __syncthreads();
    } else if (j < n) {
      const int lo = j - pool_r < 0 ? 0 : j - pool_r;
      const int hi = j + pool_r > n - 1 ? n - 1 : j + pool_r;
      for (int t = lo; t <= hi; ++t) m = fmaxf(m, s[t]);
    }
    uint32_t bin = kBins;
    if (j < n) {
      if (pout) pout[j] = m;
      const uint32_t key = float_key(m);
      keys[j] = key;
      bin = key >> 20;
    }
    hist_add(hist, bin);
  }
  if (C == 0) return;
  if (C >= n) {
    for (int j = tid; j < n; j += kSelThreads) out[j] = j;
    return;
  }
  __syncthreads();

  // 2. radix select: 12 + 12 + 8 bits
  find_bin(hist, kBins, C, warp_tot, &s_bin, &s_rem);
  uint32_t prefix = static_cast<uint32_t>(s_bin);        // top 12 bits of T
  int remaining = s_rem;
  for (int b = tid; b < kBins; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kSelThreads) {
    const int j = base + tid;
    uint32_t bin = kBins;
    if (j < n) {
      const uint32_t key = keys[j];
      if ((key >> 20) == prefix) bin = (key >> 8) & 4095u;
    }
    hist_add(hist, bin);
  }
  __syncthreads();
  find_bin(hist, kBins, remaining, warp_tot, &s_bin, &s_rem);
  prefix = (prefix << 12) | static_cast<uint32_t>(s_bin);   // top 24 bits of T
  remaining = s_rem;
  for (int b = tid; b < 256; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kSelThreads) {
    const int j = base + tid;
    uint32_t bin = kBins;
    if (j < n) {
      const uint32_t key = keys[j];
      if ((key >> 8) == prefix) bin = key & 255u;
    }
    hist_add(hist, bin);
  }
  __syncthreads();
  find_bin(hist, 256, remaining, warp_tot, &s_bin, &s_rem);
  const uint32_t T = (prefix << 8) | static_cast<uint32_t>(s_bin);
  const int take_eq = s_rem;   // keys equal to T to take, lowest index first

  // 3. ordered emission: warp w owns [w * chunk, (w + 1) * chunk)
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
  const int eq_before = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? eq : 0, warp_tot, total), 0);
  int my_eq = take_eq - eq_before;
  my_eq = my_eq < 0 ? 0 : (my_eq > eq ? eq : my_eq);
  int pos = __shfl_sync(0xffffffffu, block_exclusive_scan(lane == 0 ? gt + my_eq : 0, warp_tot, total), 0);
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

}  // namespace

size_t topk_ws_bytes(int units, int n_cand) {
  return static_cast<size_t>(units) * static_cast<size_t>(n_cand > 0 ? n_cand : 0) * sizeof(uint32_t);
}

cudaError_t launch_topk(const float* scores, int units, int n_cand, int pool_kernel, int k, int n_tail, int* idx,
                        float* pooled, void* ws, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  topk_kernel<<<units, kSelThreads, 0, stream>>>(scores, n_cand, pool_kernel / 2, k, n_tail, idx, pooled,
                                                 static_cast<uint32_t*>(ws));
  return cudaGetLastError();
}

}  // namespace spk
