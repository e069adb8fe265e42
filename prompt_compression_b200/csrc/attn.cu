// attn.cu -- prefill attention of the window and lookahead rows on tcgen05,
// emitting the rows' outputs and their input-key log-sum-exp.
//
// "Draft-based Approximate Inference for LLMs" (paper notes), section 关键设计,
// SpecKV: the input tokens and the lookahead tokens go through the target
// model's prefill together, and the importance of the input KV pairs is read
// from the attention of the last n_window input rows and the lookahead rows.
// This kernel is that attention for those rows: row i (head-local) sits at
// position n_in - n_window + i and attends causally to the keys up to it --
// the n_in input keys, then (lookahead rows only) the lookahead keys up to
// its own.  Outputs per row:
//   out   = softmax(scale q.k) V over the visible keys (bf16)
//   lse2  = log2 sum_{visible input keys} 2^(c2 q.k), c2 = scale log2(e):
//           the normaliser of the importance scores, written as the row
//           offsets the column pass (speckv_colsum) reads, so that scoring
//           after this attention needs only the column pass.
//
// Work decomposition: an item is a pair of one unit's 128-row Q tiles (A
// and B) sharing every K/V tile; a persistent CTA walks items.  Key tiles of
// 128: phase A over the input keys (tile t at key 128 t; the unit's input
// K/V tensor map ends at n_in, so the last tile's tail reads as zeros and is
// masked), then phase B over the lookahead keys (their own tensor map).
// After phase A every row's (max, sum) gives the input-key LSE.
//   warps 0-3, 4-7 : softmax of Q tile A, B; thread = query row (TMEM lane).
//               Per key tile: S (128 fp32 columns) read in two halves for the
//               row max (the second half kept in registers), lazy rescale
//               (the running max moves only when a tile's max exceeds it by
//               more than 8 in log2 units; O and the sum are rescaled then),
//               P = 2^(c2 s - m) into TMEM as bf16 pairs over columns
//               [64, 128) of the S buffer (the first half read again).
//   warp 8    : TMA producer (both Q tiles per item; K and V tiles through a
//               2-stage ring).
//   warp 9    : TMEM allocator + single-thread UMMA issuer, per key tile t:
//               O_A += P_A(t) V(t), S_A(t+1) = Q_A K(t+1)^T, O_B += P_B(t) V(t),
//               S_B(t+1) = Q_B K(t+1)^T -- each softmax group works while the
//               other group's products run, and S_x(t+1) is issued after
//               O_x's product of tile t, so O_x is quiescent once S_x(t+1)
//               has landed.  S = Q K^T takes A and B from shared memory;
//               O += P V takes A = P from TMEM and B = V from shared memory
//               in its natural [key][d] layout (MN-major), in two key halves:
//               keys 64..127 once the softmax has stored their P (it stores
//               those first), keys 0..63 once all of P is in.
// TMEM (512 columns): tile A's S at 0 and O at 128, tile B's S at 256 and O
// at 384.  No atomics: the result is deterministic.
#include <cuda_bf16.h>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "score.cuh"

namespace spk {

SPK_ERROR_READER(device_errors_attn)

namespace {

constexpr int kAttnSoftmaxWarps = 4;     // per Q tile; two groups
constexpr int kAttnProducerWarp = 8;
constexpr int kAttnMmaWarp = 9;
constexpr int kAttnThreads = 10 * 32;
constexpr float kRescaleLog2 = 8.f;    // lazy rescale threshold (P <= 2^8)
constexpr int kAttnPolyOf8 = 1;        // exponential pairs (of 8) evaluated on the FMA pipe (0, 1 and 2 within 1 %)

template <int D>
struct AttnCfg {
  static constexpr int kTileBytes = 128 * D * 2;   // 128 rows x D bf16 (Q, K or V tile)
  static constexpr int kAtoms = D / 64;            // 128-byte swizzle atoms along D
  static constexpr int kStages = 2;
  static constexpr int kSmemBytes = 1024 + 2 * kTileBytes + 2 * kStages * kTileBytes;   // Q x 2, K and V rings
  static_assert(kSmemBytes <= 227 * 1024 - 2048, "fits one CTA");
};

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled
// layout TMA writes: 128-byte rows along K (here: keys), N (here: head_dim)
// contiguous inside a row, 8-row (1024-byte) swizzle atoms stacked along K
// (stride byte offset), 64-element column blocks `lbo` bytes apart along N.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// 32 consecutive 32-bit TMEM columns of this thread's lane from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// (lo, hi) -> bf16x2 with lo in the low half: one packed conversion.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Row r (0..127) of a row-offset block: v split into three bf16 terms
// (the layout the column pass reads; see kOffBlockBytes).
__device__ __forceinline__ void attn_store_offset_row(uint8_t* block, int r, float v) {
  const __nv_bfloat16 h1 = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h1);
  const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(h2);
  const __nv_bfloat16 h3 = __float2bfloat16_rn(r2);
  const uint32_t w0 = static_cast<uint32_t>(__bfloat16_as_ushort(h1)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h2)) << 16);
  const uint32_t w1 = static_cast<uint32_t>(__bfloat16_as_ushort(h3));
  uint8_t* row = block + (r >> 3) * 256 + (r & 7) * 16;
  *reinterpret_cast<uint4*>(row) = make_uint4(w0, w1, 0u, 0u);
  *reinterpret_cast<uint4*>(row + 128) = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ int attn_site(int role, int which) { return 300 + role * 10 + which; }

}  // namespace

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap klmap,
                const __grid_constant__ CUtensorMap vlmap, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const Q_s = smem;                                   // [2 tiles]
  uint8_t* const K_s = smem + 2 * C::kTileBytes;
  uint8_t* const V_s = K_s + C::kStages * C::kTileBytes;

  // per Q tile x (0: A, 1: B): s_full[x] (S ready), p_full[x] (P written, 4
  // warps), pv_done[x] (O += P V retired), o_empty[x] (O read at item end)
  __shared__ __align__(8) uint64_t q_full, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2],
      p_half[2], p_full[2], pv_done[2], o_empty[2], done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_a = (p.n_in + 127) / 128;
  const int tiles_b = (p.n_look + 127) / 128;
  const int n_tiles = tiles_a + tiles_b;
  const int pairs = (p.row_tiles + 1) / 2;                     // items per unit: Q tiles 2 pr, 2 pr + 1
  const int n_items = p.n_items;                               // units * pairs

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_half[s], kAttnSoftmaxWarps); mbar_init(&p_full[s], kAttnSoftmaxWarps);
      mbar_init(&pv_done[s], 1); mbar_init(&o_empty[s], kAttnSoftmaxWarps);
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kAttnMmaWarp) {
    tmem_alloc(&tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == kAttnProducerWarp && lane == 0) {
    tma_prefetch_map(&qmap);
    tma_prefetch_map(&kmap);
    tma_prefetch_map(&vmap);
    if (tiles_b > 0) {
      tma_prefetch_map(&klmap);
      tma_prefetch_map(&vlmap);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  volatile int* abort_v = &abort_flag;

  if (warp == kAttnProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      uint32_t tile_count = 0;     // K/V tiles loaded by this CTA (stage = count % 2)
      int items_done = 0;
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1}, q_last = -1;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++items_done) {
        const int u = item / pairs, pr = item % pairs;
        if (!(ok = mbar_wait(&q_empty, (items_done & 1) ^ 1, abort_v, attn_site(0, 0)))) break;
        mbar_arrive_expect_tx(&q_full, 2 * C::kTileBytes);
        for (int x = 0; x < 2; ++x)
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(Q_s + x * C::kTileBytes + a * 16384, &qmap, &q_full, a * 64, (2 * pr + x) * 128, u);
        q_last = items_done & 1;
        for (int t = 0; ok && t < n_tiles; ++t, ++tile_count) {
          const int st = tile_count & 1;
          const uint32_t ph = (tile_count >> 1) & 1;
          const bool in_a = t < tiles_a;
          const int row0 = in_a ? t * 128 : (t - tiles_a) * 128;
          if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, abort_v, attn_site(0, 1)))) break;
          mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(K_s + st * C::kTileBytes + a * 16384, in_a ? &kmap : &klmap, &k_full[st], a * 64, row0, u);
          k_last[st] = static_cast<int>(ph);
          if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, abort_v, attn_site(0, 2)))) break;
          mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(V_s + st * C::kTileBytes + a * 16384, in_a ? &vmap : &vlmap, &v_full[st], a * 64, row0, u);
          v_last[st] = static_cast<int>(ph);
        }
      }
      if (!ok) {
        volatile int never = 0;
        if (q_last >= 0) mbar_wait(&q_full, q_last, &never, attn_site(0, 7), 100000000ull);
        for (int s = 0; s < 2; ++s) {
          if (k_last[s] >= 0) mbar_wait(&k_full[s], k_last[s], &never, attn_site(0, 8), 100000000ull);
          if (v_last[s] >= 0) mbar_wait(&v_full[s], v_last[s], &never, attn_site(0, 9), 100000000ull);
        }
      }
    }
  } else if (warp == kAttnMmaWarp) {
    // ------------------------------------------------------------ UMMA issuer
    // Order per key tile t: PV_A(t), S_A(t + 1), PV_B(t), S_B(t + 1), so that
    // each softmax group overlaps the other's products, and S_x(t + 1) is
    // issued after PV_x(t): when S_x(t + 1) has landed, O_x is quiescent.
    if (lane == 0) {
      bool ok = true;
      uint32_t T = 0;              // key tiles of this CTA before the current item
      int items_done = 0;
      const uint32_t idesc_s = idesc_bf16_f32(128, 128);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D) | (1u << 16);    // B (V) MN-major, N = head_dim
      auto issue_s = [&](int x, uint32_t Ti) -> bool {
        const int st = Ti & 1;
        if (x == 0 && !mbar_wait(&k_full[st], (Ti >> 1) & 1, abort_v, attn_site(1, 1))) return false;
        tc_fence_after();
        const uint64_t q_desc = sw128_kmajor_desc(smem_u32(Q_s + x * C::kTileBytes));
        const uint64_t k_desc = sw128_kmajor_desc(smem_u32(K_s + st * C::kTileBytes));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_bf16_ss(tmem_base + x * 256, q_desc + koff, k_desc + koff, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[x]);
        if (x == 1) umma_commit(&k_empty[st]);
        return true;
      };
      // O += P V in two halves: keys 64..127 as soon as the softmax has
      // stored their P (while it works on keys 0..63), then keys 0..63
      auto issue_pv = [&](int x, uint32_t Ti, int t) -> bool {
        const int st = Ti & 1;
        if (!mbar_wait(&p_half[x], Ti & 1, abort_v, attn_site(1, 2 + x))) return false;
        if (x == 0 && !mbar_wait(&v_full[st], (Ti >> 1) & 1, abort_v, attn_site(1, 6))) return false;
        // the softmax group has read the previous item's O before it is restarted
        if (t == 0 && items_done > 0 && !mbar_wait(&o_empty[x], (items_done - 1) & 1, abort_v, attn_site(1, 7 + x)))
          return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(V_s + st * C::kTileBytes);
        auto pv_steps = [&](int kk0) {
#pragma unroll
          for (int kk = kk0; kk < kk0 + 4; ++kk) {
            // one instruction spans the head_dim / 64 column blocks (lbo apart)
            const uint64_t v_desc = sw128_mnmajor_desc(v_base + kk * 2048, 16384);
            umma_bf16_ts(tmem_base + x * 256 + 128, tmem_base + x * 256 + 64 + kk * 8, v_desc, idesc_pv,
                         (t > 0 || kk != 4) ? 1u : 0u);
          }
        };
        pv_steps(4);
        if (!mbar_wait(&p_full[x], Ti & 1, abort_v, attn_site(1, 4 + x))) return false;
        tc_fence_after();
        pv_steps(0);
        umma_commit(&pv_done[x]);
        if (x == 1) umma_commit(&v_empty[st]);
        return true;
      };
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++items_done) {
        if (!(ok = mbar_wait(&q_full, items_done & 1, abort_v, attn_site(1, 0)))) break;
        if (!(ok = issue_s(0, T)) || !(ok = issue_s(1, T))) break;
        for (int t = 0; ok && t < n_tiles; ++t) {
          const uint32_t Tc = T + t;
          if (!(ok = issue_pv(0, Tc, t))) break;
          if (t + 1 < n_tiles && !(ok = issue_s(0, Tc + 1))) break;
          if (!(ok = issue_pv(1, Tc, t))) break;
          if (t + 1 < n_tiles && !(ok = issue_s(1, Tc + 1))) break;
        }
        if (!ok) break;
        umma_commit(&q_empty);
        T += n_tiles;
      }
      umma_commit(&done_bar);
      volatile int never = 0;
      mbar_wait(&done_bar, 0, &never, attn_site(1, 9), 100000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    const int x = warp >> 2;                                   // Q tile of this group (0: A, 1: B)
    const int wq = warp & 3;                                   // TMEM lane quarter
    const int r = wq * 32 + lane;                              // row within the Q tile = TMEM lane
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + x * 256;   // S; O at +128
    bool ok = true;
    uint32_t T = 0;
    int items_done = 0;
    auto wait_all = [&](uint64_t* bar, uint32_t parity, int which) -> bool {
      bool w = mbar_wait(bar, parity, abort_v, attn_site(2 + x, which));
      return __all_sync(0xffffffffu, w);
    };
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++items_done) {
      const int u = item / pairs, rb = 2 * (item % pairs) + x;   // this group's Q tile
      const int n = rb * 128 + r;                       // row within the unit
      const bool live = n < p.rows;
      const int c = p.c0 + (live ? n % p.R : 0);        // visible keys (input, then lookahead)
      float m = -INFINITY, l = 0.f, lse_in = 0.f;       // m: running max of c2 * s
      for (int t = 0; ok && t < n_tiles; ++t) {
        const uint32_t Tc = T + t;
        if (!(ok = wait_all(&s_full[x], Tc & 1, 0))) break;
        tc_fence_after();
        // keys of this tile this row sees: [0, lim)
        const bool in_a = t < tiles_a;
        const int j0 = in_a ? t * 128 : p.n_in + (t - tiles_a) * 128;
        const int j_end = in_a ? min(j0 + 128, p.n_in) : min(j0 + 128, p.n_in + p.n_look);
        const int lim = max(0, min(c, j_end) - j0);
        // S columns [0, 64) then [64, 128): the row max; the second half stays
        // in registers
        auto mask64 = [&](uint32_t (&a0)[32], uint32_t (&a1)[32], int c0) {
          if (lim < c0 + 64) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              if (c0 + k >= lim) a0[k] = __float_as_uint(-INFINITY);
              if (c0 + 32 + k >= lim) a1[k] = __float_as_uint(-INFINITY);
            }
          }
        };
        auto max64 = [&](const uint32_t (&a0)[32], const uint32_t (&a1)[32], float mx) {
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            mx = fmaxf(mx, max3f(__uint_as_float(a0[k]), __uint_as_float(a0[k + 1]),
                                 fmaxf(__uint_as_float(a0[k + 2]), __uint_as_float(a0[k + 3]))));
            mx = fmaxf(mx, max3f(__uint_as_float(a1[k]), __uint_as_float(a1[k + 1]),
                                 fmaxf(__uint_as_float(a1[k + 2]), __uint_as_float(a1[k + 3]))));
          }
          return mx;
        };
        float mx;
        uint32_t b0[32], b1[32];                         // S columns [64, 128)
        {
          uint32_t a0[32], a1[32];
          tmem_ld32(tlane, a0);
          tmem_ld32(tlane + 32, a1);
          tmem_ld_wait2(a0, a1);
          mask64(a0, a1, 0);
          mx = max64(a0, a1, -INFINITY);
        }
        tmem_ld32(tlane + 64, b0);
        tmem_ld32(tlane + 96, b1);
        tmem_ld_wait2(b0, b1);
        mask64(b0, b1, 64);
        mx = max64(b0, b1, mx);
        const float mt = mx * p.c2;
        const bool need = lim > 0 && mt > m + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m - mt) : 1.f;   // m = -inf: alpha = 0
          if (t > 0) {
            // O holds the P.V products of tiles 0 .. t-1, all retired (S(t) was issued after them)
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t o[32];
              tmem_ld32(tlane + 128 + ch * 32, o);
              tmem_ld_wait(o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(tlane + 128 + ch * 32, o);
            }
            tmem_st_wait();
          }
          if (need) {
            l *= alpha;
            m = mt;
          }
        }
        // P = 2^(c2 s - m) (masked keys: 2^-inf = 0) as bf16 pairs in TMEM
        // columns [64, 128): those of S columns [64, 128) (in registers) go to
        // [96, 128), then S columns [0, 64) are read again and theirs go to
        // [64, 96) -- every column written has been read already.  Packed
        // fp32x2 math; kAttnPolyOf8 of every 8 exponential pairs on the FMA pipe.
        const float2 c2v = f2(p.c2, p.c2), nm = f2(-m, -m);
        float2 acc2 = f2(0.f, 0.f);
        auto exp64 = [&](const uint32_t (&a0)[32], const uint32_t (&a1)[32], uint32_t (&pk)[32]) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 tt = __ffma2_rn(f2(__uint_as_float(a0[2 * k]), __uint_as_float(a0[2 * k + 1])), c2v, nm);
            const float2 e = ((k & 7) < kAttnPolyOf8) ? exp2_fma_pair(tt) : exp2_mufu_pair(tt);
            acc2 = __fadd2_rn(acc2, e);
            pk[k] = pack_bf16(e.x, e.y);
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 tt = __ffma2_rn(f2(__uint_as_float(a1[2 * k]), __uint_as_float(a1[2 * k + 1])), c2v, nm);
            const float2 e = ((k & 7) < kAttnPolyOf8) ? exp2_fma_pair(tt) : exp2_mufu_pair(tt);
            acc2 = __fadd2_rn(acc2, e);
            pk[16 + k] = pack_bf16(e.x, e.y);
          }
        };
        {
          uint32_t pk[32];
          exp64(b0, b1, pk);
          tmem_st32(tlane + 96, pk);
        }
        // keys 64..127 of P are in: their half of O += P V can start
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_half[x]);
        {
          uint32_t a0[32], a1[32];
          tmem_ld32(tlane, a0);
          tmem_ld32(tlane + 32, a1);
          tmem_ld_wait2(a0, a1);
          mask64(a0, a1, 0);
          uint32_t pk[32];
          exp64(a0, a1, pk);
          tmem_st32(tlane + 64, pk);
        }
        l += acc2.x + acc2.y;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
        if (t == tiles_a - 1) lse_in = m + lg2_approx(l);   // every input key is in
      }
      if (!ok) break;
      // ---- O of this item: after the last P.V, scale by 1 / l and store.
      // S(Tl) landed after P.V(Tl - 1) retired, so the P.V barrier's phase
      // for P.V(Tl) is the newest or the one just completed.
      const uint32_t Tl = T + n_tiles - 1;
      if (!(ok = wait_all(&pv_done[x], Tl & 1, 3))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                            (static_cast<size_t>(u) * p.rows + (live ? n : 0)) * D;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tlane + 128 + ch * 32, o);
        tmem_ld_wait(o);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            dst[v4] = w;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[x]);
      if (p.lse2 != nullptr && live) p.lse2[static_cast<size_t>(u) * p.rows + n] = lse_in;
      if (p.off_blocks != nullptr && rb < p.row_tiles)
        attn_store_offset_row(p.off_blocks + (static_cast<size_t>(u) * p.row_tiles + rb) * kOffBlockBytes, r,
                              live ? -lse_in / p.c2 : -1e30f);
      T += n_tiles;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kAttnMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int D>
static cudaError_t attn_launch_one(const CUtensorMap (&maps)[5], const AttnParams& p, int grid,
                                   cudaStream_t stream) {
  using C = AttnCfg<D>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  attn_kernel<D><<<grid, kAttnThreads, C::kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

cudaError_t launch_attn(int head_dim, const CUtensorMap (&maps)[5], const AttnParams& p, int grid,
                        cudaStream_t stream) {
  if (head_dim == 128) return attn_launch_one<128>(maps, p, grid, stream);
  if (head_dim == 64) return attn_launch_one<64>(maps, p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace spk
