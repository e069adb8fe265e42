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
// Short caches: a persistent CTA per SM streams its units (below); long
// caches: one CTA per (batch, layer, KV head) unit.  Warp w takes the 32-row
// blocks w, w + W, ... of a unit.  A block's K and V rows are copied into the warp's
// shared-memory slot (cp.async, 16-byte chunks placed with an XOR swizzle so
// that ldmatrix reads are conflict-free); with more blocks than warps each
// warp keeps two slots, the next block in flight while one is used.  Both
// contractions run on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate), the g <= 8 query heads of the unit being the n = 8 side:
//   logits  S^T[t][h] = sum_d K[t][d] Q[h][d]        A = K rows (ldmatrix),
//                                                     B = Q (registers)
//   output  O^T[d][h] += sum_t V^T[d][t] P^T[t][h]   A = V^T (ldmatrix.trans),
//                                                     B = P^T (movmatrix of the
//                                                     logits' layout)
// P = 2^(c2 s - m) (online softmax per head, log2 domain, fp32) enters the
// second product as two bf16 terms, P = hi + lo with hi = bf16(P), lo =
// bf16(P - hi), so the weights keep 16 significant bits (relative error
// <= 2^-17) while V stays exact.  The warps' states are merged in a fixed
// order at the end, so results are bitwise reproducible.  Every K and V byte
// is read once: bound by HBM bandwidth.
#include <cuda_bf16.h>

#include "common.cuh"
#include "score.cuh"

namespace spk {
namespace {

constexpr int kDecMaxWarps = 12;
constexpr int kDecSmemBudget = 200 * 1024;   // stage slots of one CTA

// 16-byte chunk `ch` of row `row` (rows of D bf16) in a swizzled slot
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return static_cast<uint32_t>(row * (D * 2) + ((ch ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// d += a * b, m16n8k16, bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// One block of MT * 16 rows of a unit (K at shared address ks, V at vs,
// swizzled): its logits for the 8 query-head columns, the online-softmax
// update of (m, l) for this thread's heads 2gc and 2gc + 1, and
// O^T += V^T P^T.
template <int D, int MT>
__device__ __forceinline__ void block_update(uint32_t ks, uint32_t vs, int t0, int n_kv, float c2,
                                             const uint32_t (&bq)[D / 16][2], float (&o)[D / 16][4], float& m0,
                                             float& m1, float& l0, float& l1) {
  constexpr int KS = D / 16;
  const int lane = threadIdx.x & 31;
  const int gr = lane >> 2;
  // logits: two 16-row m-tiles; ldmatrix x4 of A: matrices (rows 0-7 | 8-15) x (chunk 2s | 2s+1)
  // (even and odd k-steps accumulate separately: two chains of KS / 2)
  float sc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    const int arow = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int s = 0; s < KS; s += 2) {
      uint32_t a[4], b[4];
      ldsm_x4(ks + swz<D>(arow, 2 * s + (lane >> 4)), a);
      ldsm_x4(ks + swz<D>(arow, 2 * s + 2 + (lane >> 4)), b);
      mma_bf16(sa, a, bq[s][0], bq[s][1]);
      mma_bf16(sb, b, bq[s + 1][0], bq[s + 1][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[mt][e] = sa[e] + sb[e];
  }
  // online softmax per head over the block's rows (this thread: rows
  // t0 + 16mt + gr (+8), heads 2gc and 2gc + 1); lanes sharing gc hold
  // the other rows
  float z[MT][4];
  float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = t0 + mt * 16 + gr + (e >> 1) * 8;
      z[mt][e] = t < n_kv ? sc[mt][e] * c2 : -INFINITY;
    }
    bm0 = fmaxf(bm0, fmaxf(z[mt][0], z[mt][2]));
    bm1 = fmaxf(bm1, fmaxf(z[mt][1], z[mt][3]));
  }
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, o2));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, o2));
  }
  const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);   // finite: row t0 is valid
  const float al0 = ex2_approx(m0 - mn0), al1 = ex2_approx(m1 - mn1);   // 0 while m = -inf
  m0 = mn0;
  m1 = mn1;
  float s0 = 0.f, s1 = 0.f;
  uint32_t phi[MT][2], plo[MT][2];   // per m-tile: rows gr | gr + 8, heads (2gc, 2gc + 1) as bf16 pairs
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    float p[4];
    p[0] = ex2_approx(z[mt][0] - mn0);
    p[1] = ex2_approx(z[mt][1] - mn1);
    p[2] = ex2_approx(z[mt][2] - mn0);
    p[3] = ex2_approx(z[mt][3] - mn1);
    s0 += p[0] + p[2];
    s1 += p[1] + p[3];
    float h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = bf16_round(p[e]);
    phi[mt][0] = pack_bf16(h[0], h[1]);
    phi[mt][1] = pack_bf16(h[2], h[3]);
    plo[mt][0] = pack_bf16(p[0] - h[0], p[1] - h[1]);
    plo[mt][1] = pack_bf16(p[2] - h[2], p[3] - h[3]);
  }
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, o2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o2);
  }
  l0 = fmaf(l0, al0, s0);
  l1 = fmaf(l1, al1, s1);
#pragma unroll
  for (int j = 0; j < KS; ++j) {
    o[j][0] *= al0;
    o[j][1] *= al1;
    o[j][2] *= al0;
    o[j][3] *= al1;
  }
  // P^T B fragments: the 8x8 blocks (rows t, cols h) transposed
  uint32_t bh[MT][2], bl[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    bh[mt][0] = movm_t(phi[mt][0]);
    bh[mt][1] = movm_t(phi[mt][1]);
    bl[mt][0] = movm_t(plo[mt][0]);
    bl[mt][1] = movm_t(plo[mt][1]);
  }
  // O^T += V^T P^T: m-tile j over d, k-step mt over the block's rows;
  // ldmatrix x4 .trans: matrices (rows 0-7 | 8-15 of the k-step) x (chunk 2j | 2j+1)
  const int vrow = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      uint32_t a[4];
      ldsm_x4_t(vs + swz<D>(mt * 16 + vrow, 2 * j + ((lane >> 3) & 1)), a);
      mma_bf16(o[j], a, bh[mt][0], bh[mt][1]);
      mma_bf16(o[j], a, bl[mt][0], bl[mt][1]);
    }
  }
}

// S slots per warp, each holding one 32-row block: K then V (32 * D bf16 each).
template <int D, int S>
__global__ void __launch_bounds__(kDecMaxWarps * 32, 1)
    decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                  float* __restrict__ out, int g, int n_kv, float c2) {
  constexpr int kRowB = D * 2;                 // bytes of a row
  constexpr int kHalfB = 32 * kRowB;           // K (or V) of a block
  constexpr int kSlotB = 2 * kHalfB;
  constexpr int KS = D / 16;                   // k-steps over d; m-tiles over d
  extern __shared__ __align__(128) uint8_t dec_smem[];   // [warps][S][slot]; reused by the merge
  __shared__ float m_s[kDecMaxWarps][8], l_s[kDecMaxWarps][8];

  const int unit = blockIdx.x;   // (b * layers + l) * hkv + h; its query heads are rows unit*g .. unit*g+g-1
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, gc = lane & 3;     // fragment row group, column pair

  // B fragments of Q (k = d, n = head): b0 = Q[gr][16s + 2gc, +1], b1 = +8
  uint32_t bq[KS][2];
  {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(q + static_cast<size_t>(unit) * g * D);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      bq[s][0] = gr < g ? __ldg(q32 + gr * (D / 2) + 8 * s + gc) : 0u;
      bq[s][1] = gr < g ? __ldg(q32 + gr * (D / 2) + 8 * s + gc + 4) : 0u;
    }
  }
  // output state: O^T[d][h] fragments (m-tile j: d = 16j + gr (+8); h = 2gc, 2gc + 1)
  float o[KS][4];
#pragma unroll
  for (int j = 0; j < KS; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads 2gc, 2gc + 1

  const uint8_t* kb = reinterpret_cast<const uint8_t*>(k + static_cast<size_t>(unit) * n_kv * D);
  const uint8_t* vb = reinterpret_cast<const uint8_t*>(v + static_cast<size_t>(unit) * n_kv * D);
  uint8_t* my = dec_smem + static_cast<size_t>(warp) * S * kSlotB;
  const uint32_t my_s = smem_u32(my);
  const int nblk = (n_kv + 31) / 32;

  // block b -> slot: rows past n_kv copy the last row (finite values, weight 0)
  auto issue = [&](int b, int slot) {
    if (b < nblk) {
      uint8_t* dk = my + slot * kSlotB;
      uint8_t* dv = dk + kHalfB;
      constexpr int kChunks = 32 * kRowB / 16;
#pragma unroll
      for (int i = 0; i < kChunks / 32; ++i) {
        const int c = i * 32 + lane;
        const int row = c / (kRowB / 16), ch = c % (kRowB / 16);
        const int t = min(b * 32 + row, n_kv - 1);
        const size_t src = static_cast<size_t>(t) * kRowB + ch * 16;
        cp_async16(dk + swz<D>(row, ch), kb + src);
        cp_async16(dv + swz<D>(row, ch), vb + src);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < S; ++i) issue(warp + i * warps, i);

  for (int it = 0;; ++it) {
    const int b = warp + it * warps;
    if (b >= nblk) break;
    const int slot = it % S;
    cp_async_wait<S - 1>();
    __syncwarp();
    const uint32_t ks = my_s + slot * kSlotB, vs = ks + kHalfB;
    const int t0 = b * 32;

    block_update<D, 2>(ks, vs, t0, n_kv, c2, bq, o, m0, m1, l0, l1);
    __syncwarp();                                     // the slot is free
    issue(b + S * warps, slot);
  }
  cp_async_wait<0>();

  // merge the warps' states in a fixed order (acc_s reuses the slots)
  __syncthreads();
  float* acc_s = reinterpret_cast<float*>(dec_smem);   // [warps][8][D]
#pragma unroll
  for (int j = 0; j < KS; ++j) {
    const int d0 = 16 * j + gr;
    acc_s[(warp * 8 + 2 * gc) * D + d0] = o[j][0];
    acc_s[(warp * 8 + 2 * gc + 1) * D + d0] = o[j][1];
    acc_s[(warp * 8 + 2 * gc) * D + d0 + 8] = o[j][2];
    acc_s[(warp * 8 + 2 * gc + 1) * D + d0 + 8] = o[j][3];
  }
  if (gr == 0) {
    m_s[warp][2 * gc] = m0;
    m_s[warp][2 * gc + 1] = m1;
    l_s[warp][2 * gc] = l0;
    l_s[warp][2 * gc + 1] = l1;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < g * D; x += blockDim.x) {
    const int h = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < warps; ++w) M = fmaxf(M, m_s[w][h]);
    float L = 0.f, A = 0.f;
    for (int w = 0; w < warps; ++w) {
      if (m_s[w][h] == -INFINITY) continue;   // a warp that saw no row
      const float f = ex2_approx(m_s[w][h] - M);
      L = fmaf(l_s[w][h], f, L);
      A = fmaf(acc_s[(w * 8 + h) * D + c], f, A);
    }
    out[(static_cast<size_t>(unit) * g + h) * D + c] = A / L;
  }
}

// Persistent streaming over units, for short caches (up to 4 blocks of 16
// rows per warp and unit): one or two CTAs per SM take the units
// blockIdx.x, + gridDim.x, ...; warp w takes the 16-row blocks w, w + W, ... of each,
// and its two slots keep the next block in flight across unit boundaries, so
// the loads of the next unit overlap the merge of the current one (the merge
// state has its own shared memory).  Q fragments of the next unit are
// fetched one unit ahead.  16-row blocks keep each warp's dependent chain
// short and let ten warps share an SM's shared memory.
constexpr int kStreamMaxWarps = 10;
constexpr int kStreamRows = 16;
constexpr int kStreamMaxBlocks = 4 * kStreamMaxWarps;   // 16-row blocks

template <int D>
__global__ void __launch_bounds__(kStreamMaxWarps * 32, 1)
    decode_stream_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                         const uint16_t* __restrict__ v, float* __restrict__ out, int units, int g, int n_kv,
                         float c2) {
  constexpr int kRowB = D * 2;
  constexpr int kHalfB = kStreamRows * kRowB;
  constexpr int kSlotB = 2 * kHalfB;
  constexpr int KS = D / 16;
  extern __shared__ __align__(128) uint8_t dec_smem[];   // [W][2][slot], then the merge state [W][8][D] fp32
  __shared__ float m_s[kStreamMaxWarps][8], l_s[kStreamMaxWarps][8];

  const int W = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, gc = lane & 3;
  const int nblk = (n_kv + kStreamRows - 1) / kStreamRows;
  const int J = (nblk + W - 1) / W;                       // block positions per warp and unit
  const int cta = blockIdx.x, ctas = gridDim.x;
  const int n_my = units > cta ? (units - 1 - cta) / ctas + 1 : 0;
  const int n_items = n_my * J;
  uint8_t* my = dec_smem + static_cast<size_t>(warp) * 2 * kSlotB;
  float* acc_s = reinterpret_cast<float*>(dec_smem + static_cast<size_t>(W) * 2 * kSlotB);

  // item = (unit position kk, block position j) -> slot; rows past n_kv copy the last row
  auto issue = [&](int item, int slot) {
    if (item < n_items) {
      const int kk = item / J, b = warp + (item % J) * W;
      if (b < nblk) {
        const size_t base = static_cast<size_t>(cta + kk * ctas) * n_kv * kRowB;
        const uint8_t* kb = reinterpret_cast<const uint8_t*>(k) + base;
        const uint8_t* vb = reinterpret_cast<const uint8_t*>(v) + base;
        uint8_t* dk = my + slot * kSlotB;
        uint8_t* dv = dk + kHalfB;
        constexpr int kChunks = kStreamRows * kRowB / 16;
        const bool full = (b + 1) * kStreamRows <= n_kv;
#pragma unroll
        for (int i = 0; i < kChunks / 32; ++i) {
          const int c = i * 32 + lane;
          const int row = c / (kRowB / 16), ch = c % (kRowB / 16);
          const int t = full ? b * kStreamRows + row : min(b * kStreamRows + row, n_kv - 1);
          const size_t src = static_cast<size_t>(t) * kRowB + ch * 16;
          cp_async16(dk + swz<D>(row, ch), kb + src);
          cp_async16(dv + swz<D>(row, ch), vb + src);
        }
      }
    }
    cp_async_commit();
  };
  auto load_q = [&](int kk, uint32_t (&bq)[KS][2]) {
    const bool ok = kk < n_my && gr < g;
    const uint32_t* q32 =
        reinterpret_cast<const uint32_t*>(q + static_cast<size_t>(ok ? cta + kk * ctas : 0) * g * D);
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) {
      bq[s2][0] = ok ? __ldg(q32 + gr * (D / 2) + 8 * s2 + gc) : 0u;
      bq[s2][1] = ok ? __ldg(q32 + gr * (D / 2) + 8 * s2 + gc + 4) : 0u;
    }
  };

  issue(0, 0);
  issue(1, 1);
  uint32_t bq[KS][2], bq_next[KS][2];
  load_q(0, bq);
  int item = 0;
  for (int kk = 0; kk < n_my; ++kk) {
    load_q(kk + 1, bq_next);
    float o[KS][4];
#pragma unroll
    for (int j = 0; j < KS; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    for (int j = 0; j < J; ++j, ++item) {
      const int slot = item & 1;
      cp_async_wait<1>();                                 // this item's copies
      __syncwarp();
      const int b = warp + j * W;
      if (b < nblk) {
        const uint32_t ks = smem_u32(my + slot * kSlotB);
        block_update<D, 1>(ks, ks + kHalfB, b * kStreamRows, n_kv, c2, bq, o, m0, m1, l0, l1);
      }
      __syncwarp();                                       // the slot is free
      issue(item + 2, slot);
    }
    // merge the warps' states for unit cta + kk * ctas, in a fixed order
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      const int d0 = 16 * j + gr;
      acc_s[(warp * 8 + 2 * gc) * D + d0] = o[j][0];
      acc_s[(warp * 8 + 2 * gc + 1) * D + d0] = o[j][1];
      acc_s[(warp * 8 + 2 * gc) * D + d0 + 8] = o[j][2];
      acc_s[(warp * 8 + 2 * gc + 1) * D + d0 + 8] = o[j][3];
    }
    if (gr == 0) {
      m_s[warp][2 * gc] = m0;
      m_s[warp][2 * gc + 1] = m1;
      l_s[warp][2 * gc] = l0;
      l_s[warp][2 * gc + 1] = l1;
    }
    __syncthreads();
    // per head: each warp's factor 2^(m_w - M) (0 for a warp that saw no
    // row; the M's warp is never empty) and 1 / L, once
    if (threadIdx.x < 8) {
      const int h = threadIdx.x;
      float M = -INFINITY;
      for (int w = 0; w < W; ++w) M = fmaxf(M, m_s[w][h]);
      float L = 0.f;
      for (int w = 0; w < W; ++w) {
        const float f = m_s[w][h] == -INFINITY ? 0.f : ex2_approx(m_s[w][h] - M);
        m_s[w][h] = f;
        L = fmaf(l_s[w][h], f, L);
      }
      l_s[0][h] = L;
    }
    __syncthreads();
    const size_t unit = static_cast<size_t>(cta + kk * ctas);
    for (int x = threadIdx.x; x < g * D; x += blockDim.x) {
      const int h = x / D, c = x % D;
      float A = 0.f;
      for (int w = 0; w < W; ++w) A = fmaf(acc_s[(w * 8 + h) * D + c], m_s[w][h], A);
      out[(unit * g + h) * D + c] = A / l_s[0][h];
    }
    __syncthreads();                                      // the merge state is free
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) {
      bq[s2][0] = bq_next[s2][0];
      bq[s2][1] = bq_next[s2][1];
    }
  }
  cp_async_wait<0>();
}

template <int D, int S>
cudaError_t launch_ds(const void* q, const void* k, const void* v, float* out, int units, int g, int n_kv,
                      float c2, int warps, cudaStream_t stream) {
  const int smem = warps * S * (32 * D * 2 * 2);
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e =
        cudaFuncSetAttribute(decode_kernel<D, S>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemBudget);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  decode_kernel<D, S><<<units, warps * 32, smem, stream>>>(static_cast<const uint16_t*>(q),
                                                         static_cast<const uint16_t*>(k),
                                                         static_cast<const uint16_t*>(v), out, g, n_kv, c2);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_stream(const void* q, const void* k, const void* v, float* out, int units, int g, int n_kv,
                          float c2, cudaStream_t stream) {
  constexpr int kSlotB = kStreamRows * D * 2 * 2;
  constexpr int kSmemMax = kStreamMaxWarps * (2 * kSlotB + 8 * D * 4);
  static_assert(kSmemMax <= 227 * 1024, "streaming slots and merge state fit");
  static thread_local int configured_device = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(decode_stream_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  // Up to 4 block positions per warp.  With at most 5 warps (20 blocks) two
  // CTAs share an SM (their per-unit merges overlap each other's loads);
  // otherwise up to kStreamMaxWarps warps, one CTA per SM.
  const int blocks = (n_kv + kStreamRows - 1) / kStreamRows;
  constexpr int kPairWarps = 5;
  int per = (blocks + kPairWarps - 1) / kPairWarps;                 // block positions per warp
  int ctas_per_sm = 2;
  if (per > 4) {
    per = (blocks + kStreamMaxWarps - 1) / kStreamMaxWarps;
    ctas_per_sm = 1;
  }
  const int warps = (blocks + per - 1) / per;
  const int smem = warps * (2 * kSlotB + 8 * D * 4);
  static_assert(2 * kPairWarps * (2 * kSlotB + 8 * D * 4) <= 227 * 1024, "two CTAs of five warps share an SM");
  const int grid = units < ctas_per_sm * sms ? units : ctas_per_sm * sms;
  decode_stream_kernel<D><<<grid, warps * 32, smem, stream>>>(static_cast<const uint16_t*>(q),
                                                              static_cast<const uint16_t*>(k),
                                                              static_cast<const uint16_t*>(v), out, units, g, n_kv,
                                                              c2);
  return cudaGetLastError();
}

// Short caches (up to kStreamMaxBlocks blocks): the persistent streaming
// kernel.  Longer caches: one CTA per unit, two slots per warp (the next
// block in flight while one is used), as many warps as the slots' budget
// allows.
template <int D>
cudaError_t launch_d(const void* q, const void* k, const void* v, float* out, int units, int g, int n_kv,
                     float c2, cudaStream_t stream) {
  constexpr int kSlotB = 32 * D * 2 * 2;
  static_assert(kDecMaxWarps * kSlotB <= kDecSmemBudget, "one slot per warp fits");
  static_assert(32 * D * 2 * 2 >= 8 * D * 4, "a warp's slot holds its merge state");
  if ((n_kv + kStreamRows - 1) / kStreamRows <= kStreamMaxBlocks)
    return launch_stream<D>(q, k, v, out, units, g, n_kv, c2, stream);
  int warps = kDecSmemBudget / (2 * kSlotB);
  warps = warps > 8 ? 8 : warps;
  return launch_ds<D, 2>(q, k, v, out, units, g, n_kv, c2, warps, stream);
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, float* out, int units, int g,
                          int head_dim, int n_kv, float c2, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  if (g < 1 || g > 8) return cudaErrorInvalidValue;
  if (head_dim == 128) return launch_d<128>(q, k, v, out, units, g, n_kv, c2, stream);
  if (head_dim == 64) return launch_d<64>(q, k, v, out, units, g, n_kv, c2, stream);
  return cudaErrorInvalidValue;
}

}  // namespace spk
