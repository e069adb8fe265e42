// select.cu -- max-pooling and deterministic top-k selection with a kept tail.
//
// "Draft-based Approximate Inference for LLMs" (paper notes): section 关键设计
// keeps the top-C_max KV pairs plus the window; section 损失函数 / 训练策略
// smooths SpecPC scores with local pooling so that kept tokens form runs.
//
// One CTA per row of candidates:
//   1. pooled[j] = max of scores over the clipped window [j-r, j+r]; the
//      pooled values are stored as order-preserving 32-bit keys.
//   2. radix select (4 passes of 8 bits, most significant first) finds the
//      exact key T of the C-th largest value and how many keys equal to T
//      must be taken; histograms are built with warp-aggregated shared atomics.
//   3. emission: each thread owns a contiguous run of indices; two block-wide
//      prefix sums (keys equal to T, then selected keys) give every thread its
//      output offset, so the indices come out ascending with ties resolved
//      lowest index first -- no sort is needed.
#include "common.cuh"
#include "score.cuh"

namespace spk {
namespace {

constexpr int kSelThreads = 1024;

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
    int w = warp_tot[lane];
    int wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    warp_tot[lane] = wx - w;        // exclusive warp offsets
    if (lane == 31) warp_tot[32] = wx;
  }
  __syncthreads();
  const int out = warp_tot[warp] + x - v;
  total = warp_tot[32];
  __syncthreads();
  return out;
}

__global__ void __launch_bounds__(kSelThreads, 1)
    topk_kernel(const float* __restrict__ scores, int n_cand, int pool_r, int k, int n_tail, int* __restrict__ idx,
                float* __restrict__ pooled, uint32_t* __restrict__ keys_ws) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  __shared__ int warp_tot[33];

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
  uint32_t* keys = keys_ws + static_cast<size_t>(u) * n;
  float* pout = pooled ? pooled + static_cast<size_t>(u) * n : nullptr;

  // 1. pooling -> keys
  for (int j = tid; j < n; j += kSelThreads) {
    const int lo = j - pool_r < 0 ? 0 : j - pool_r;
    const int hi = j + pool_r > n - 1 ? n - 1 : j + pool_r;
    float m = s[lo];
    for (int t = lo + 1; t <= hi; ++t) m = fmaxf(m, s[t]);
    if (pout) pout[j] = m;
    keys[j] = float_key(m);
  }
  if (C == 0) return;
  if (C >= n) {
    for (int j = tid; j < n; j += kSelThreads) out[j] = j;
    return;
  }
  __syncthreads();

  // 2. radix select of the C-th largest key
  uint32_t prefix = 0, pmask = 0;
  int remaining = C;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = tid; b < 256; b += kSelThreads) hist[b] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kSelThreads) {
      const int j = base + tid;
      uint32_t digit = 256;
      if (j < n) {
        const uint32_t key = keys[j];
        if ((key & pmask) == prefix) digit = (key >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (digit != 256 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
    }
    __syncthreads();
    if (tid == 0) {
      int cum = 0;
      for (int b = 255; b >= 0; --b) {
        const int h = static_cast<int>(hist[b]);
        if (cum + h >= remaining) {
          prefix |= static_cast<uint32_t>(b) << shift;
          remaining -= cum;
          break;
        }
        cum += h;
      }
      s_prefix = prefix;
      s_remaining = remaining;
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    pmask |= 255u << shift;
  }
  const uint32_t T = prefix;
  const int take_eq = remaining;   // keys equal to T to take, lowest index first

  // 3. ordered emission
  const int seg = (n + kSelThreads - 1) / kSelThreads;
  const int beg = tid * seg < n ? tid * seg : n;
  const int end = beg + seg < n ? beg + seg : n;
  int gt = 0, eq = 0;
  for (int j = beg; j < end; ++j) {
    const uint32_t key = keys[j];
    gt += key > T;
    eq += key == T;
  }
  int total;
  const int eq_before = block_exclusive_scan(eq, warp_tot, total);
  int my_eq = take_eq - eq_before;
  my_eq = my_eq < 0 ? 0 : (my_eq > eq ? eq : my_eq);
  int pos = block_exclusive_scan(gt + my_eq, warp_tot, total);
  for (int j = beg; j < end; ++j) {
    const uint32_t key = keys[j];
    if (key > T) {
      out[pos++] = j;
    } else if (key == T && my_eq > 0) {
      out[pos++] = j;
      --my_eq;
    }
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
