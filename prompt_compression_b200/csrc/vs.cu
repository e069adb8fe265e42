// vs.cu -- Vertical-Slash sparse prefill attention on tcgen05.
//
// "Draft-based Approximate Inference for LLMs" (paper notes), section
// 损失函数 / 训练策略: SpecKV runs the target model's prefill with
// Vertical-Slash sparse attention (the pattern of the cited sparse-attention
// work).  Per unit (batch element, layer, KV head) the pattern is a sorted
// set V of key columns and a sorted set S of diagonals (offsets o = p - j);
// the query row at position p attends to the keys j <= p with j in V, or
// p - j in S, or j = p (the token itself):
//   out = softmax_j(scale q.k_j) . v_j over those keys (bf16), lse2 (optional,
//   log2 domain) of the same sum.
// Query rows are the last n_q positions of the n-token sequence, every query
// head of the unit's GQA group.
//
// Work decomposition: an item is a pair of query heads of one unit's GQA
// group (heads 2 hp and 2 hp + 1) over one 128-row block (positions
// p0 .. p0 + 127).  The two heads have the same rows, hence the same key
// tiles and the same masks: they share every K/V tile, and two softmax
// warpgroups (one per head) work in ping-pong, each while the other head's
// products run.  The item's keys come in 128-key tiles of two kinds:
//   slash tiles    -- tiles of K/V that a slash diagonal (or the self
//                     diagonal) crosses for some row of the item: tile t is
//                     crossed iff some o in S u {0} lies in
//                     [p0 - 128 t - 127, p_last - 128 t]; found by one walk
//                     over S from the diagonal tile down;
//   vertical tiles -- the vertical keys <= p_last, gathered beforehand into a
//                     contiguous [units][n_v][d] buffer (kv_compact).
// Masks are exact: in a slash tile key j is visible iff j <= p and (j = p or
// j in V or p - j in S), from bitmaps of V and S in shared memory (one 32-bit
// word per 32 keys, the slash word bit-reversed); in a vertical tile a key is
// visible iff j <= p and its K/V tile was not a slash tile of the item (there
// it was already counted).  The pipeline is the prefill attention's: a TMA
// producer warp (both heads' Q tiles, then the K/V tiles), a single-thread
// UMMA issuer (per tile: O_A += P_A V, S_A(next), O_B += P_B V, S_B(next);
// S = Q K^T from shared memory, O += P V with P in TMEM as bf16 and V
// MN-major from shared memory, keys 64..127 as soon as their P is stored) and eight softmax warps (thread = row; S read
// in 64-column halves; lazy rescale of O when the running max moves by more
// than 2^8).  Every role derives the same tile sequence.
#include <cuda_bf16.h>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "score.cuh"

namespace spk {

SPK_ERROR_READER(device_errors_vs)

namespace {

constexpr int kVsGroupWarps = 4;       // softmax warps per head of the pair (two groups)
constexpr int kVsProducerWarp = 8;
constexpr int kVsMmaWarp = 9;
constexpr int kVsThreads = 10 * 32;
constexpr float kVsRescale = 8.f;
constexpr int kVsPolyOf8 = 0;          // exponential pairs (of 8) on the FMA pipe: none (the kernel is ALU bound; measured best)

template <int D>
struct VsCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kAtoms = D / 64;
  static constexpr int kStages = 2;
  static constexpr int kBitWords = kVsMaxN / 32;
  static constexpr int kSmemBytes =
      1024 + 2 * kTileBytes + 2 * kStages * kTileBytes + 2 * kBitWords * 4 + kVsMaxVert * 4;   // Q x 2, K and V rings
  static_assert(kSmemBytes <= 227 * 1024 - 2048, "fits one CTA");
};

__device__ __forceinline__ uint64_t vs_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void vs_tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
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

// 16 consecutive 32-bit TMEM columns of this thread's lane from registers.
__device__ __forceinline__ void vs_tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// (lo, hi) -> bf16x2 with lo in the low half: one packed conversion.
__device__ __forceinline__ uint32_t vs_pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ int vs_site(int role, int which) { return 400 + role * 10 + which; }


// Marks in `tb` (one bit per 128-key tile) the slash tiles of an item whose
// rows sit at positions p0 .. p_last (p_last - p0 < 128): tile t (0 <= t <=
// p_last / 128) is crossed iff some offset o in S u {0} lies in
// [p0 - 128 t - 127, p_last - 128 t], i.e. t in [floor((p0 - o) / 128),
// floor((p_last - o) / 128)] -- at most two tiles per offset.  Thread `tid`
// of `nthreads` takes every nthreads-th offset (the loads are independent);
// the caller clears the words first and synchronises after.
__device__ __forceinline__ void mark_slash_tiles(uint32_t* tb, const int* __restrict__ S, int n_s, int p0, int p_last,
                                                 int tid, int nthreads) {
  const int t_top = p_last >> 7;
  for (int i = tid; i <= n_s; i += nthreads) {
    const int o = i < n_s ? __ldg(S + i) : 0;
    const int lo = max((p0 - o) >> 7, 0), hi = min((p_last - o) >> 7, t_top);
    for (int t = lo; t <= hi; ++t) atomicOr(&tb[t >> 5], 1u << (t & 31));
  }
}

// Walks the set bits of a tile bitmap from the highest down (the order in
// which every role takes an item's slash tiles).
struct TileWalk {
  int w;
  uint32_t m;
  __device__ __forceinline__ TileWalk(const uint32_t* tb, int t_top) : w(t_top >> 5), m(tb[t_top >> 5]) {}
  __device__ __forceinline__ int next(const uint32_t* tb) {
    while (m == 0u) {
      if (--w < 0) return -1;
      m = tb[w];
    }
    const int b = 31 - __clz(m);
    m &= ~(1u << b);
    return w * 32 + b;
  }
};

// Number of entries of the ascending array x[0, n) that are <= v, by the
// whole warp: 32 probes per step narrow the answer's range 32-fold, so
// n <= 32^k takes k dependent loads.  Every lane returns the count.
__device__ __forceinline__ int warp_count_le(const int* __restrict__ x, int n, int v, int lane) {
  int lo = 0, len = n;                  // the count lies in [lo, lo + len]
  while (len > 32) {
    const int step = (len + 31) >> 5;
    const int i = lo + lane * step;
    const bool le = i < lo + len && __ldg(x + i) <= v;
    const int c = __popc(__ballot_sync(0xffffffffu, le));   // probes <= v: a prefix
    if (c == 0) return lo;
    const int nlo = lo + (c - 1) * step + 1;
    len = min(lo + c * step, lo + len) - nlo;
    lo = nlo;
  }
  const bool le = lane < len && __ldg(x + lo + lane) <= v;
  return lo + __popc(__ballot_sync(0xffffffffu, le));
}

// 32 bits of a bitmap starting at bit o (bits below 0 and at or above
// n_bits read as 0).
__device__ __forceinline__ uint32_t bits32(const uint32_t* bm, int n_words, int o) {
  if (o <= -32) return 0u;
  if (o < 0) return n_words > 0 ? bm[0] << (-o) : 0u;
  const int w = o >> 5, sh = o & 31;
  const uint32_t lo = w < n_words ? bm[w] : 0u;
  if (sh == 0) return lo;
  const uint32_t hi = w + 1 < n_words ? bm[w + 1] : 0u;
  return (lo >> sh) | (hi << (32 - sh));
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kVsThreads, 1)
    vs_attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kvmap,
                   const __grid_constant__ CUtensorMap vvmap, const VsParams p) {
  using C = VsCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const Q_s = smem;                                    // [2 heads]
  uint8_t* const K_s = smem + 2 * C::kTileBytes;
  uint8_t* const V_s = K_s + C::kStages * C::kTileBytes;
  uint32_t* const vbits = reinterpret_cast<uint32_t*>(V_s + C::kStages * C::kTileBytes);   // V as a bitmap
  uint32_t* const sbits = vbits + C::kBitWords;                                           // S as a bitmap
  int* const vidx_s = reinterpret_cast<int*>(sbits + C::kBitWords);                      // V, ascending

  // per Q tile x (0: A, 1: B): s_full[x], p_full[x] (4 warps), pv_done[x], o_empty[x] (4 warps)
  __shared__ __align__(8) uint64_t q_full, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2],
      p_half[2], p_full[2], pv_done[2], o_empty[2], done_bar, soft_bar;
  __shared__ uint32_t slash_tiles[kVsMaxN / 128 / 32];   // the softmax warps' item: its slash tiles
  __shared__ uint32_t prod_tiles[kVsMaxN / 128 / 32];    // the producer's item
  __shared__ uint32_t mma_tiles[kVsMaxN / 128 / 32];     // the UMMA issuer's item
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n = p.n;
  const int n_words = (n + 31) >> 5;
  const int hpairs = (p.g + 1) / 2;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_half[s], kVsGroupWarps); mbar_init(&p_full[s], kVsGroupWarps);
      mbar_init(&pv_done[s], 1); mbar_init(&o_empty[s], kVsGroupWarps);
    }
    mbar_init(&done_bar, 1);
    mbar_init(&soft_bar, 2 * kVsGroupWarps);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kVsMmaWarp) {
    tmem_alloc(&tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == kVsProducerWarp && lane == 0) {
    tma_prefetch_map(&qmap);
    tma_prefetch_map(&kmap);
    tma_prefetch_map(&vmap);
    if (p.n_v > 0) {
      tma_prefetch_map(&kvmap);
      tma_prefetch_map(&vvmap);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  volatile int* abort_v = &abort_flag;

  // item -> (unit, head pair, row block); rows' positions p0 .. p_last; the
  // pair's query heads 2 hp and 2 hp + 1 of the group share every key tile
  // and every mask
  auto item_geom = [&](int item, int& u, int& hp, int& rb, int& p0, int& p_last) {
    rb = item % p.row_blocks;
    const int hu = item / p.row_blocks;   // u * hpairs + hp
    u = hu / hpairs;
    hp = hu % hpairs;
    p0 = n - p.n_q + rb * 128;
    p_last = n - p.n_q + min(rb * 128 + 127, p.n_q - 1);
  };
  // tiles of an item: its slash tiles (marked in tb), then ceil(cv / 128)
  // vertical tiles (cv = vertical keys <= p_last); whole warp, every lane
  // returns the counts
  auto warp_item_tiles = [&](uint32_t* tb, int u, int p0, int p_last, int& n_slash, int& cv) {
    const int nw = ((p_last >> 7) >> 5) + 1;
    for (int w = lane; w < nw; w += 32) tb[w] = 0u;
    __syncwarp();
    mark_slash_tiles(tb, p.slash + static_cast<size_t>(u) * p.n_s, p.n_s, p0, p_last, lane, 32);
    __syncwarp();
    n_slash = 0;
    for (int w = 0; w < nw; ++w) n_slash += __popc(tb[w]);
    cv = p.n_v > 0 ? warp_count_le(p.vert + static_cast<size_t>(u) * p.n_v, p.n_v, p_last, lane) : 0;
    return n_slash + (cv + 127) / 128;
  };

  if (warp > kVsMmaWarp) {
    // (no other warps)
  } else if (warp == kVsProducerWarp) {
    // ------------------------------------------------------------ producer
    // (the whole warp derives each item's tiles; lane 0 issues the copies)
    {
      bool ok = true;
      uint32_t tile_count = 0;
      int items_done = 0;
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1}, q_last = -1;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++items_done) {
        int u, hp, rb, p0, p_last;
        item_geom(item, u, hp, rb, p0, p_last);
        int n_slash, cv;
        const int n_tiles = warp_item_tiles(prod_tiles, u, p0, p_last, n_slash, cv);
        if (lane == 0) do {
        if (!(ok = mbar_wait(&q_empty, (items_done & 1) ^ 1, abort_v, vs_site(0, 0)))) break;
        mbar_arrive_expect_tx(&q_full, 2 * C::kTileBytes);
        for (int x = 0; x < 2; ++x) {
          // a missing second head (odd g) loads the next head's rows (or zeros): never stored
          const int qh = u * p.g + 2 * hp + x;
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(Q_s + x * C::kTileBytes + a * 16384, &qmap, &q_full, a * 64, rb * 128, qh);
        }
        q_last = items_done & 1;
        TileWalk walk(prod_tiles, p_last >> 7);
        for (int i = 0; ok && i < n_tiles; ++i, ++tile_count) {
          const int st = tile_count & 1;
          const uint32_t ph = (tile_count >> 1) & 1;
          const bool slash = i < n_slash;
          const int row0 = slash ? 128 * walk.next(prod_tiles) : 128 * (i - n_slash);
          if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, abort_v, vs_site(0, 1)))) break;
          mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(K_s + st * C::kTileBytes + a * 16384, slash ? &kmap : &kvmap, &k_full[st], a * 64, row0, u);
          k_last[st] = static_cast<int>(ph);
          if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, abort_v, vs_site(0, 2)))) break;
          mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
          for (int a = 0; a < C::kAtoms; ++a)
            tma_load_3d(V_s + st * C::kTileBytes + a * 16384, slash ? &vmap : &vvmap, &v_full[st], a * 64, row0, u);
          v_last[st] = static_cast<int>(ph);
        }
        } while (false);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0 && !ok) {
        volatile int never = 0;
        if (q_last >= 0) mbar_wait(&q_full, q_last, &never, vs_site(0, 7), 100000000ull);
        for (int s = 0; s < 2; ++s) {
          if (k_last[s] >= 0) mbar_wait(&k_full[s], k_last[s], &never, vs_site(0, 8), 100000000ull);
          if (v_last[s] >= 0) mbar_wait(&v_full[s], v_last[s], &never, vs_site(0, 9), 100000000ull);
        }
      }
    }
  } else if (warp == kVsMmaWarp) {
    // ------------------------------------------------------------ UMMA issuer
    // Order per key tile t: O_A += P_A V(t), S_A(t+1), O_B += P_B V(t), S_B(t+1)
    // (each softmax group works while the other's products run; S_x(t+1)
    // follows O_x's product of tile t, so O_x is quiescent once it lands).
    // (the whole warp derives each item's tile count; lane 0 issues)
    {
      bool ok = true;
      uint32_t T = 0;
      int items_done = 0;
      const uint32_t idesc_s = idesc_bf16_f32(128, 128);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D) | (1u << 16);    // B (V) MN-major, N = head_dim
      auto issue_s = [&](int x, uint32_t Ti) -> bool {
        const int st = Ti & 1;
        if (x == 0 && !mbar_wait(&k_full[st], (Ti >> 1) & 1, abort_v, vs_site(1, 1))) return false;
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
        if (!mbar_wait(&p_half[x], Ti & 1, abort_v, vs_site(1, 2 + x))) return false;
        if (x == 0 && !mbar_wait(&v_full[st], (Ti >> 1) & 1, abort_v, vs_site(1, 6))) return false;
        if (t == 0 && items_done > 0 && !mbar_wait(&o_empty[x], (items_done - 1) & 1, abort_v, vs_site(1, 7 + x)))
          return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(V_s + st * C::kTileBytes);
        auto pv_steps = [&](int kk0) {
#pragma unroll
          for (int kk = kk0; kk < kk0 + 4; ++kk) {
            // one instruction spans the head_dim / 64 column blocks (lbo apart)
            const uint64_t v_desc = vs_mnmajor_desc(v_base + kk * 2048, 16384);
            umma_bf16_ts(tmem_base + x * 256 + 128, tmem_base + x * 256 + 64 + kk * 8, v_desc, idesc_pv,
                         (t > 0 || kk != 4) ? 1u : 0u);
          }
        };
        pv_steps(4);
        if (!mbar_wait(&p_full[x], Ti & 1, abort_v, vs_site(1, 4 + x))) return false;
        tc_fence_after();
        pv_steps(0);
        umma_commit(&pv_done[x]);
        if (x == 1) umma_commit(&v_empty[st]);
        return true;
      };
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++items_done) {
        int u, hp, rb, p0, p_last;
        item_geom(item, u, hp, rb, p0, p_last);
        int n_slash, cv;
        const int n_tiles = warp_item_tiles(mma_tiles, u, p0, p_last, n_slash, cv);
        if (lane == 0) do {
          if (!(ok = mbar_wait(&q_full, items_done & 1, abort_v, vs_site(1, 0)))) break;
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
        } while (false);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        T += n_tiles;
      }
      if (lane == 0) {
        umma_commit(&done_bar);
        volatile int never = 0;
        mbar_wait(&done_bar, 0, &never, vs_site(1, 9), 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    const int x = warp >> 2;                            // head of the pair (Q tile)
    const int wq = warp & 3;
    const int tid = threadIdx.x;                        // 0 .. 255 over both groups
    const int r = wq * 32 + lane;                       // row within the Q tile = TMEM lane
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + x * 256;   // S; O at +128
    bool ok = true;
    uint32_t T = 0;
    int items_done = 0, loaded_unit = -1;
    auto wait_all = [&](uint64_t* bar, uint32_t parity, int which) -> bool {
      bool w = mbar_wait(bar, parity, abort_v, vs_site(2 + x, which));
      return __all_sync(0xffffffffu, w);
    };
    // the eight softmax warps meet (their shared-memory writes before it are
    // visible after it); a bounded wait, so an aborted CTA cannot strand a warp
    uint32_t soft_phase = 0;
    auto softmax_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&soft_bar);
      const bool w = wait_all(&soft_bar, soft_phase, 4);
      soft_phase ^= 1u;
      return w;
    };
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++items_done) {
      int u, hp, rb, p0, p_last;
      item_geom(item, u, hp, rb, p0, p_last);
      // this unit's pattern as bitmaps (and V as a list), and the item's
      // slash tiles as a bitmap
      if (!(ok = softmax_sync())) break;                // the previous item is done with them
      const int tb_words = ((p_last >> 7) >> 5) + 1;
      for (int w = tid; w < tb_words; w += 256) slash_tiles[w] = 0u;
      const bool new_unit = u != loaded_unit;
      if (new_unit)
        for (int w = tid; w < n_words; w += 256) { vbits[w] = 0u; sbits[w] = 0u; }
      if (!(ok = softmax_sync())) break;
      mark_slash_tiles(slash_tiles, p.slash + static_cast<size_t>(u) * p.n_s, p.n_s, p0, p_last, tid, 256);
      if (new_unit) {
        const int* vg = p.vert + static_cast<size_t>(u) * p.n_v;
        const int* sg = p.slash + static_cast<size_t>(u) * p.n_s;
        for (int i = tid; i < p.n_v; i += 256) {
          const int j = __ldg(vg + i);
          vidx_s[i] = j;
          if (j >= 0 && j < n) atomicOr(&vbits[j >> 5], 1u << (j & 31));
          else record_error(SPK_DEVERR_INDEX, u);
        }
        for (int i = tid; i < p.n_s; i += 256) {
          const int o = __ldg(sg + i);
          if (o >= 0 && o < n) atomicOr(&sbits[o >> 5], 1u << (o & 31));
          else record_error(SPK_DEVERR_INDEX, u);
        }
        loaded_unit = u;
      }
      if (!(ok = softmax_sync())) break;
      int n_slash = 0;
      for (int w = 0; w < tb_words; ++w) n_slash += __popc(slash_tiles[w]);
      const int cv = p.n_v > 0 ? warp_count_le(p.vert + static_cast<size_t>(u) * p.n_v, p.n_v, p_last, lane) : 0;
      const int n_tiles = n_slash + (cv + 127) / 128;

      const int h = 2 * hp + x;                         // head of the group
      const int qh = u * p.g + h;
      const int i_row = rb * 128 + r;
      const bool live = i_row < p.n_q && h < p.g;
      const int pos = i_row < p.n_q ? n - p.n_q + i_row : n - 1;
      TileWalk walk(slash_tiles, p_last >> 7);          // this role's walk over the slash tiles
      float m = -INFINITY, l = 0.f;
      for (int t = 0; ok && t < n_tiles; ++t) {
        const uint32_t Tc = T + t;
        const bool slash = t < n_slash;
        int j0 = 0;
        if (slash) {
          j0 = walk.next(slash_tiles) * 128;
        }
        // visibility of the tile's 128 keys for this row, 32 per word
        uint32_t vis[4];
        if (slash) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int jc = j0 + 32 * c;
            const int rel = pos - jc;                   // key jc + b is causal iff b <= rel
            const uint32_t causal = rel < 0 ? 0u : (rel >= 31 ? 0xffffffffu : ((2u << rel) - 1u));
            const uint32_t self = (rel >= 0 && rel < 32) ? (1u << rel) : 0u;
            const uint32_t vw = (jc >> 5) < n_words ? vbits[jc >> 5] : 0u;
            const uint32_t sw = __brev(bits32(sbits, n_words, pos - jc - 31));
            vis[c] = (vw | sw | self) & causal;
          }
        } else {
          const int base = 128 * (t - n_slash);         // gathered rows of this vertical tile
          const int cnt = min(128, cv - base);
          __syncwarp();
          // keys of slash tiles were counted there; vertical keys <= pos
          // only.  The warp's rows are the consecutive positions pos0 + lane
          // (rows past n_q are never stored), and the tile's keys ascend, so
          // the keys <= pos of a 32-key chunk are a prefix of it, of length
          // (keys < pos0) + (keys in [pos0, pos0 + lane]).
          const int pos0 = __shfl_sync(0xffffffffu, pos, 0);
          const uint32_t upto = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int xx = 32 * c + lane;
            bool okc = false;
            int dj = 1 << 30;                           // key - pos0 (past the tile: never visible)
            if (xx < cnt) {
              const int j = vidx_s[base + xx];
              okc = j >= 0 && j < n && !((slash_tiles[j >> 12] >> ((j >> 7) & 31)) & 1u);
              dj = j - pos0;
            }
            const uint32_t dedupe = __ballot_sync(0xffffffffu, okc);
            const int below = __popc(__ballot_sync(0xffffffffu, dj < 0));
            const uint32_t near = __reduce_or_sync(0xffffffffu, (dj >= 0 && dj < 32) ? (1u << dj) : 0u);
            const int k = below + __popc(near & upto);   // keys of the chunk <= pos0 + lane
            const uint32_t pre = k >= 32 ? 0xffffffffu : ((1u << k) - 1u);
            vis[c] = dedupe & pre;
          }
        }
        if (!(ok = wait_all(&s_full[x], Tc & 1, 0))) break;
        tc_fence_after();
        // S columns [0, 64) then [64, 128), masked: the row max
        // (a word every lane sees whole -- the common case in vertical
        // tiles -- needs no select).  A masked word goes back to TMEM, so
        // the second pass over S reads it masked.
        auto mask64 = [&](uint32_t (&a0)[32], uint32_t (&a1)[32], uint32_t v0, uint32_t v1, uint32_t col) {
          if (__any_sync(0xffffffffu, v0 != 0xffffffffu)) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (!((v0 >> k) & 1u)) a0[k] = __float_as_uint(-INFINITY);
            vs_tmem_st32(col, a0);
          }
          if (__any_sync(0xffffffffu, v1 != 0xffffffffu)) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (!((v1 >> k) & 1u)) a1[k] = __float_as_uint(-INFINITY);
            vs_tmem_st32(col + 32, a1);
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
        float mx = -INFINITY;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t a0[32], a1[32];
          tmem_ld32(tlane + 64 * hh, a0);
          tmem_ld32(tlane + 64 * hh + 32, a1);
          tmem_ld_wait2(a0, a1);
          mask64(a0, a1, hh ? vis[2] : vis[0], hh ? vis[3] : vis[1], tlane + 64 * hh);
          mx = max64(a0, a1, mx);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");   // the masked words have landed
        const float mt = mx * p.c2;
        const bool need = mx != -INFINITY && mt > m + kVsRescale;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m - mt) : 1.f;
          if (t > 0) {
            // O holds the P.V products of tiles 0 .. t-1, all retired (S(t) was issued after them)
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t o[32];
              tmem_ld32(tlane + 128 + ch * 32, o);
              tmem_ld_wait(o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              vs_tmem_st32(tlane + 128 + ch * 32, o);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          }
          if (need) {
            l *= alpha;
            m = mt;
          }
        }
        // P = 2^(c2 s - m) into TMEM columns [64, 128) of the S buffer: S
        // columns [64, 128) are read again and theirs go to [96, 128), then
        // those of S columns [0, 64) to [64, 96) -- every column written has
        // been read.  Masked keys (s = -inf) give 0; a row that has seen no
        // key yet (m = -inf) has only masked keys here (with kVsPolyOf8 > 0
        // the FMA-pipe exponential would turn a masked key into 2^-126
        // instead of 0: far below the rounding of the sum and of O, and
        // wiped by the rescale when the row sees its first key).
        const float mm = m == -INFINITY ? 0.f : m;
        const float2 c2v = f2(p.c2, p.c2), nm = f2(-mm, -mm);
        float2 acc2 = f2(0.f, 0.f);
        // 32 S values -> 16 packed P words at TMEM column `col`
        auto exp32 = [&](const uint32_t (&a)[32], uint32_t col) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 tt = __ffma2_rn(f2(__uint_as_float(a[2 * k]), __uint_as_float(a[2 * k + 1])), c2v, nm);
            const float2 e = ((k & 7) < kVsPolyOf8) ? exp2_fma_pair(tt) : exp2_mufu_pair(tt);
            acc2 = __fadd2_rn(acc2, e);
            pk[k] = vs_pack_bf16(e.x, e.y);
          }
          vs_tmem_st16(col, pk);
        };
#pragma unroll 1
        for (int hh = 1; hh >= 0; --hh) {
          uint32_t a0[32], a1[32];
          tmem_ld32(tlane + 64 * hh, a0);
          tmem_ld32(tlane + 64 * hh + 32, a1);
          tmem_ld_wait2(a0, a1);
          exp32(a0, tlane + 64 + 32 * hh);                // masked by the first pass
          exp32(a1, tlane + 64 + 32 * hh + 16);
          if (hh == 1) {
            // keys 64..127 of P are in: their half of O += P V can start
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_half[x]);
          }
        }
        l += acc2.x + acc2.y;
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      // S(Tl) landed after P.V(Tl - 1) retired: the P.V barrier's phase for
      // P.V(Tl) is the newest or the one just completed
      const uint32_t Tl = T + n_tiles - 1;
      if (!(ok = wait_all(&pv_done[x], Tl & 1, 3))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                            (static_cast<size_t>(live ? qh : 0) * p.n_q + (live ? i_row : 0)) * D;
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
            w.x = vs_pack_bf16(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = vs_pack_bf16(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = vs_pack_bf16(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = vs_pack_bf16(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            dst[v4] = w;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[x]);
      if (p.lse2 != nullptr && live) p.lse2[static_cast<size_t>(qh) * p.n_q + i_row] = m + lg2_approx(l);
      T += n_tiles;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kVsMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int D>
static cudaError_t vs_launch_one(const CUtensorMap (&maps)[5], const VsParams& p, int grid, cudaStream_t stream) {
  using C = VsCfg<D>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e =
        cudaFuncSetAttribute(vs_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  vs_attn_kernel<D><<<grid, kVsThreads, C::kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

cudaError_t launch_vs_attn(int head_dim, const CUtensorMap (&maps)[5], const VsParams& p, int grid,
                           cudaStream_t stream) {
  if (head_dim == 128) return vs_launch_one<128>(maps, p, grid, stream);
  if (head_dim == 64) return vs_launch_one<64>(maps, p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace spk
