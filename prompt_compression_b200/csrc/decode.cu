// decode.cu -- decode attention over a compacted KV cache.
//
// "Draft-based Approximate Inference for LLMs" (paper notes): section 整体框架
// (the target model runs on the compressed KV cache, which is where the
// compute and memory saving comes from) and section 关键设计, SpecKV (the
// cache keeps the top-C_max KV pairs and the window).  For one new query token
// per attention head:
//   out[qh] = sum_t softmax_t(scale * q[qh] . k[t]) * v[t]
// over the n_kv rows of the head's KV head (GQA: query head qh reads KV head
// qh / g), e.g. the k_out / v_out that kv_compact leaves.
//
// One CTA (8 warps) per (batch, layer, KV head) unit.  Warp w takes rows
// t = 4w.., in blocks of 4 rows every 32 (so each block's K and V rows are
// independent loads in flight together); lane l holds elements
// [l * d/32, (l + 1) * d/32) of every row, so a row is one coalesced 128- or
// 256-byte load.  For each of the g query heads the warp keeps an online
// softmax state (running max in the log2 domain, running sum, and its lanes'
// slice of the weighted V sum).  At the end the 8 warps' states are merged
// in a fixed order, so results are bitwise reproducible.  Every K and V byte
// is read once: the kernel is bound by HBM bandwidth.
#include <cuda_bf16.h>

#include "common.cuh"
#include "score.cuh"

namespace spk {
namespace {

constexpr int kDecWarps = 8;
constexpr int kDecRowsPerIter = 4;   // rows a warp has in flight per iteration

template <int D>
struct RowSlice;   // one lane's d/32 bf16 elements of a row
template <>
struct RowSlice<128> {
  using T = uint2;   // 4 bf16
  static constexpr int kN = 4;
};
template <>
struct RowSlice<64> {
  using T = uint32_t;   // 2 bf16
  static constexpr int kN = 2;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__device__ __forceinline__ void unpack(const typename RowSlice<D>::T& r, float (&x)[RowSlice<D>::kN]) {
  if constexpr (D == 128) {
    x[0] = bf16_lo(r.x);
    x[1] = bf16_hi(r.x);
    x[2] = bf16_lo(r.y);
    x[3] = bf16_hi(r.y);
  } else {
    x[0] = bf16_lo(r);
    x[1] = bf16_hi(r);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32)
    decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                  float* __restrict__ out, int n_kv, float c2) {
  using S = RowSlice<D>;
  constexpr int E = S::kN;
  __shared__ float m_s[kDecWarps][G], l_s[kDecWarps][G];
  __shared__ float acc_s[kDecWarps][G][D];

  const int unit = blockIdx.x;   // (b * layers + l) * hkv + h
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this unit's query heads are G consecutive rows of q: unit * G .. unit * G + G - 1
  float qf[G][E];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const typename S::T r =
        reinterpret_cast<const typename S::T*>(q + (static_cast<size_t>(unit) * G + h) * D)[lane];
    unpack<D>(r, qf[h]);
  }
  float m[G], l[G], acc[G][E];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
  }
  const typename S::T* kr = reinterpret_cast<const typename S::T*>(k + static_cast<size_t>(unit) * n_kv * D);
  const typename S::T* vr = reinterpret_cast<const typename S::T*>(v + static_cast<size_t>(unit) * n_kv * D);

  for (int t0 = warp * kDecRowsPerIter; t0 < n_kv; t0 += kDecWarps * kDecRowsPerIter) {
    typename S::T kv_k[kDecRowsPerIter], kv_v[kDecRowsPerIter];
#pragma unroll
    for (int i = 0; i < kDecRowsPerIter; ++i) {
      const int t = t0 + i < n_kv ? t0 + i : t0;   // rows past the end repeat a valid row (masked below)
      kv_k[i] = __ldcs(kr + static_cast<size_t>(t) * 32 + lane);
      kv_v[i] = __ldcs(vr + static_cast<size_t>(t) * 32 + lane);
    }
#pragma unroll
    for (int i = 0; i < kDecRowsPerIter; ++i) {
      float kf[E], vf[E];
      unpack<D>(kv_k[i], kf);
      unpack<D>(kv_v[i], vf);
      const bool valid = t0 + i < n_kv;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(qf[h][e], kf[e], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (!valid) continue;
        const float z = s * c2;                       // log2-domain logit
        const float mn = fmaxf(m[h], z);
        const float alpha = ex2_approx(m[h] - mn);    // 0 on the first row (m = -inf)
        const float pz = ex2_approx(z - mn);
        l[h] = l[h] * alpha + pz;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = fmaf(acc[h][e], alpha, pz * vf[e]);
        m[h] = mn;
      }
    }
  }
  // merge the warps' states in a fixed order
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) {
      m_s[warp][h] = m[h];
      l_s[warp][h] = l[h];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc_s[warp][h][lane * E + e] = acc[h][e];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += kDecWarps * 32) {
    const int h = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, m_s[w][h]);
    float L = 0.f, A = 0.f;
    for (int w = 0; w < kDecWarps; ++w) {
      if (m_s[w][h] == -INFINITY) continue;   // a warp that saw no row
      const float f = ex2_approx(m_s[w][h] - M);
      L = fmaf(l_s[w][h], f, L);
      A = fmaf(acc_s[w][h][c], f, A);
    }
    out[(static_cast<size_t>(unit) * G + h) * D + c] = A / L;
  }
}

template <int D, int G>
cudaError_t launch_g(const void* q, const void* k, const void* v, float* out, int units, int n_kv, float c2,
                     cudaStream_t stream) {
  decode_kernel<D, G><<<units, kDecWarps * 32, 0, stream>>>(static_cast<const uint16_t*>(q),
                                                            static_cast<const uint16_t*>(k),
                                                            static_cast<const uint16_t*>(v), out, n_kv, c2);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const void* q, const void* k, const void* v, float* out, int units, int g, int n_kv,
                     float c2, cudaStream_t stream) {
  switch (g) {
    case 1: return launch_g<D, 1>(q, k, v, out, units, n_kv, c2, stream);
    case 2: return launch_g<D, 2>(q, k, v, out, units, n_kv, c2, stream);
    case 3: return launch_g<D, 3>(q, k, v, out, units, n_kv, c2, stream);
    case 4: return launch_g<D, 4>(q, k, v, out, units, n_kv, c2, stream);
    case 5: return launch_g<D, 5>(q, k, v, out, units, n_kv, c2, stream);
    case 6: return launch_g<D, 6>(q, k, v, out, units, n_kv, c2, stream);
    case 7: return launch_g<D, 7>(q, k, v, out, units, n_kv, c2, stream);
    case 8: return launch_g<D, 8>(q, k, v, out, units, n_kv, c2, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, float* out, int units, int g,
                          int head_dim, int n_kv, float c2, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  if (head_dim == 128) return launch_d<128>(q, k, v, out, units, g, n_kv, c2, stream);
  if (head_dim == 64) return launch_d<64>(q, k, v, out, units, g, n_kv, c2, stream);
  return cudaErrorInvalidValue;
}

}  // namespace spk
