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
// One CTA per (batch, layer, KV head) unit, one warp per 32-row block (up to
// 16 warps; with more blocks each warp takes blocks w, w + warps, ...).  For
// its block a warp first issues the copy of the 32 V rows into its own
// shared-memory buffer (cp.async, 16 bytes per lane per copy), then reads
// the K rows: lane l owns row t0 + l, requests the whole row at once and
// dots it with the g query rows held in shared memory (broadcast reads), so
// no cross-lane reduction is needed per row.  K and V of the block are thus
// in flight together.  The block's max and sum per query head take one warp
// reduction each (online softmax: log2-domain running max and sum); for the
// weighted V sum lane l owns elements [l * d/32, (l + 1) * d/32) of every V
// row, read from shared memory.  At the end the warps' states are merged in
// a fixed order, so results are bitwise reproducible.  Every K and V byte is
// read once: the kernel is bound by HBM bandwidth.
#include <cuda_bf16.h>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "score.cuh"

namespace spk {
namespace {

// Up to 12 warps.  A short cache (at most one 32-row block per warp) reads
// each K row in two halves, so that groups of up to 6 query heads fit 80
// registers and two CTAs (one unit each) share an SM; a long cache (many
// blocks per warp, where the exposed latency of the second half would
// repeat block after block) keeps the whole row in flight, one CTA per SM.
constexpr int kDecMaxWarps = 12;
template <int G, bool LONG>
constexpr int dec_blocks_per_sm() { return (G <= 6 && !LONG) ? 2 : 1; }

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

template <int D, int G, bool LONG>
__global__ void __launch_bounds__(kDecMaxWarps * 32, dec_blocks_per_sm<G, LONG>())
    decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                  float* __restrict__ out, int n_kv, float c2) {
  using S = RowSlice<D>;
  constexpr int E = S::kN;                    // V elements per lane
  constexpr int kBlockBytes = 32 * D * 2;     // one warp's V block
  extern __shared__ __align__(16) uint8_t dec_smem[];   // [warps][kBlockBytes]; reused by the merge
  __shared__ __align__(16) float q_s[G][D];
  __shared__ float p_s[kDecMaxWarps][G][32];
  __shared__ float m_s[kDecMaxWarps][G], l_s[kDecMaxWarps][G];

  const int unit = blockIdx.x;   // (b * layers + l) * hkv + h; its query heads are rows unit*G .. unit*G+G-1
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < G * D; i += blockDim.x)
    q_s[i / D][i % D] = __uint_as_float(static_cast<uint32_t>(q[static_cast<size_t>(unit) * G * D + i]) << 16);
  __syncthreads();

  float m[G], l[G], acc[G][E];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
  }
  const uint16_t* kr = k + static_cast<size_t>(unit) * n_kv * D;
  const uint8_t* vbytes = reinterpret_cast<const uint8_t*>(v + static_cast<size_t>(unit) * n_kv * D);
  uint8_t* vbuf = dec_smem + warp * kBlockBytes;

  for (int t0 = warp * 32; t0 < n_kv; t0 += warps * 32) {
    const int rows = n_kv - t0 < 32 ? n_kv - t0 : 32;
    // the block's V rows -> shared memory, in flight while K is read
    {
      const uint8_t* src = vbytes + static_cast<size_t>(t0) * D * 2;
      const int chunks = rows * (D * 2 / 16);
      for (int c = lane; c < chunks; c += 32) cp_async16(vbuf + c * 16, src + c * 16);
      cp_async_commit();
    }
    const int t = t0 + lane;
    const bool valid = t < n_kv;
    // logits of this lane's row for every query head of the group: the K
    // row in two halves (D/16 16-byte pieces in flight at once), packed
    // fp32x2 multiply-adds
    const uint4* krow = reinterpret_cast<const uint4*>(kr + static_cast<size_t>(valid ? t : t0) * D);
    float2 z2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) z2[h] = f2(0.f, 0.f);
    constexpr int kParts = LONG ? 1 : 2;               // pieces of the row in flight at once
    constexpr int kPer = D / 8 / kParts;
#pragma unroll
    for (int half = 0; half < kParts; ++half) {
      uint4 kbuf[kPer];
#pragma unroll
      for (int c = 0; c < kPer; ++c) kbuf[c] = __ldg(krow + half * kPer + c);
#pragma unroll
      for (int c = 0; c < kPer; ++c) {
        const uint4 kk = kbuf[c];
        const float2 k0 = f2(bf16_lo(kk.x), bf16_hi(kk.x)), k1 = f2(bf16_lo(kk.y), bf16_hi(kk.y));
        const float2 k2 = f2(bf16_lo(kk.z), bf16_hi(kk.z)), k3 = f2(bf16_lo(kk.w), bf16_hi(kk.w));
        const int e0 = (half * kPer + c) * 8;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 qa = *reinterpret_cast<const float4*>(&q_s[h][e0]);
          const float4 qb = *reinterpret_cast<const float4*>(&q_s[h][e0 + 4]);
          z2[h] = __ffma2_rn(f2(qa.x, qa.y), k0, z2[h]);
          z2[h] = __ffma2_rn(f2(qa.z, qa.w), k1, z2[h]);
          z2[h] = __ffma2_rn(f2(qb.x, qb.y), k2, z2[h]);
          z2[h] = __ffma2_rn(f2(qb.z, qb.w), k3, z2[h]);
        }
      }
    }
    float z[G];
#pragma unroll
    for (int h = 0; h < G; ++h) z[h] = z2[h].x + z2[h].y;
    // online softmax over the block, per query head
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float zz = valid ? z[h] * c2 : -INFINITY;   // log2-domain logit
      float bm = zz;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
      const float mn = fmaxf(m[h], bm);
      const float alpha = ex2_approx(m[h] - mn);   // 0 while m = -inf
      const float pz = valid ? ex2_approx(zz - mn) : 0.f;
      float bs = pz;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
      l[h] = fmaf(l[h], alpha, bs);
      m[h] = mn;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[h][e] *= alpha;
      p_s[warp][h][lane] = pz;
    }
    cp_async_wait<0>();
    __syncwarp();
    // weighted V sum over the block's rows (from shared memory); lane owns E elements of a row
    const typename S::T* vs = reinterpret_cast<const typename S::T*>(vbuf);
#pragma unroll 4
    for (int j = 0; j < rows; ++j) {
      float vf[E];
      unpack<D>(vs[j * 32 + lane], vf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pj = p_s[warp][h][j];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const float2 a = __ffma2_rn(f2(pj, pj), f2(vf[e], vf[e + 1]), f2(acc[h][e], acc[h][e + 1]));
          acc[h][e] = a.x;
          acc[h][e + 1] = a.y;
        }
      }
    }
    __syncwarp();   // the buffer and p_s are free for the next block
  }
  // merge the warps' states in a fixed order (acc_s reuses the V buffers)
  __syncthreads();
  float* acc_s = reinterpret_cast<float*>(dec_smem);   // [warps][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) {
      m_s[warp][h] = m[h];
      l_s[warp][h] = l[h];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc_s[(warp * G + h) * D + lane * E + e] = acc[h][e];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) {
    const int h = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < warps; ++w) M = fmaxf(M, m_s[w][h]);
    float L = 0.f, A = 0.f;
    for (int w = 0; w < warps; ++w) {
      if (m_s[w][h] == -INFINITY) continue;   // a warp that saw no row
      const float f = ex2_approx(m_s[w][h] - M);
      L = fmaf(l_s[w][h], f, L);
      A = fmaf(acc_s[(w * G + h) * D + c], f, A);
    }
    out[(static_cast<size_t>(unit) * G + h) * D + c] = A / L;
  }
}

template <int D, int G, bool LONG>
cudaError_t launch_gl(const void* q, const void* k, const void* v, float* out, int units, int n_kv, float c2,
                      int warps, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, LONG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDecMaxWarps * 32 * D * 2);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  decode_kernel<D, G, LONG><<<units, warps * 32, warps * 32 * D * 2, stream>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), out, n_kv,
      c2);
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_g(const void* q, const void* k, const void* v, float* out, int units, int n_kv, float c2,
                     cudaStream_t stream) {
  // one warp per 32-row block, up to 12; each warp's V block in shared memory
  static_assert(32 * D * 2 >= G * D * 4, "a warp's V buffer holds its merge state");
  const int blocks = (n_kv + 31) / 32;
  const int warps = blocks < 1 ? 1 : (blocks > kDecMaxWarps ? kDecMaxWarps : blocks);
  if (blocks <= kDecMaxWarps) return launch_gl<D, G, false>(q, k, v, out, units, n_kv, c2, warps, stream);
  return launch_gl<D, G, true>(q, k, v, out, units, n_kv, c2, warps, stream);
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
