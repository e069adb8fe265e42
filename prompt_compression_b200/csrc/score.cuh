// score.cuh -- parameters shared by the scoring kernel and its host launcher.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spk {

enum ScoreMode : int {
  MODE_LSE = 0,        // pass 1: per query row, lse2 = log2 sum_j 2^(c2 q.k_j) over visible keys
  MODE_COLSUM = 1,     // pass 2, SpecKV: per key, sum over the unit's rows of 2^(c2 q.k - lse2)
  MODE_COLSUM_PC = 2,  // pass 2, SpecPC: per key, weighted layer/row mean per query head, max over heads
};

constexpr int kRowsMax = 2048;   // query rows per unit (g * rows-per-head)

// Row-offset block of one 128-row B tile: the column passes need
// t = c2 * q.k - lse2[row] for every logit.  Instead of adding lse2 in the
// epilogue, each query row carries v = -lse2[row] / c2 split into three bf16
// terms (h1 + h2 + h3 = v to ~2^-24 relative), and one extra UMMA K-step
// against a keys-side block of ones adds them to the accumulator, which then
// holds q.k + v and only needs the scale c2.  Layout: K-major, no swizzle,
// 8-row x 16-byte core matrices: row r's K-chunk c (8 bf16) at
// (r / 8) * 256 + c * 128 + (r % 8) * 16; chunk 0 = (h1, h2, h3, 0 x 5),
// chunk 1 = 0.  Rows past the unit's rows get v = -1e30 (their terms vanish).
constexpr int kOffBlockBytes = 4096;
constexpr int kHeadsMax = 32;    // SpecPC: query heads per layer

struct ScoreParams {
  // geometry of a unit (one batch element, layer >= l_skip, KV head)
  int head_dim;
  int n_in;          // input keys per unit
  int rows;          // query rows per unit = g * R, ordered [query head][row]
  int R;             // rows per query head
  uint32_t R_mul;    // ceil(2^32 / R) for R > 1: n / R = umulhi(n, R_mul), exact while n * R < 2^32
  int c0;            // head-local row i sees keys [0, min(n_in, c0 + i))
  float c2;          // scale * log2(e)
  // unit u = (b * layers_used + l') * hkv + h  ->  tensor coordinate
  // (b * layers_total + l_skip + l') * hkv + h of the [B*L*Hkv][rows|n_in][d] views
  int hkv;
  int layers_used;
  int layers_total;
  int l_skip;
  int n_units;
  // work decomposition
  int n_items;       // persistent-loop items
  int n_blocks;      // items per unit (LSE: 256-row blocks) or per batch/unit (256-key blocks)
  // buffers
  float* lse2;       // pass 1 without off_blocks: lse2[u * lse_stride + row] (rows only)
  int lse_stride;    // floats between units in lse2
  // Row offsets between the passes, as operand blocks of one extra UMMA
  // K-step (see kOffBlockBytes): pass 1 writes them (when non-null), the
  // column passes read them.  off_tiles = 128-row tiles per unit.
  uint8_t* off_blocks;
  int off_tiles;
  float* out0;       // SpecKV scores [n_units][n_pre] or SpecPC scores [batch][n_in]
  float* out1;       // SpecKV window mass [n_units][n_in - n_pre] (nullable)
  int n_pre;         // prefix keys that are scored
  int n_cols;        // keys whose column sums are written
  const float* row_weights;  // SpecPC row weights [R] (LSE folds -log2(w_i / norm) into lse2)
  // SpecPC column pass: the (KV head, layer) segments of a key block are
  // split into seg_groups groups (one item each); with more than one group
  // every item writes per-query-head partial sums [item][hq][256] to part,
  // and launch_specpc_merge reduces them.
  int seg_groups;
  float* part;
};

cudaError_t launch_score(int mode, int head_dim, const CUtensorMap& amap, const CUtensorMap& bmap,
                         const ScoreParams& p, int grid, cudaStream_t stream);

// Device error words, one per translation unit that records errors (read,
// and cleared when `clear`, by spk_device_error()).
cudaError_t device_errors_api(int* code, int* site, bool clear);
cudaError_t device_errors_score(int* code, int* site, bool clear);
cudaError_t device_errors_attn(int* code, int* site, bool clear);
cudaError_t device_errors_vs(int* code, int* site, bool clear);
cudaError_t device_errors_compact(int* code, int* site, bool clear);
// scores[b][j] = max_qh sum_g part[(b * n_blocks + j / 256) * groups + g][qh][j % 256]
cudaError_t launch_specpc_merge(const float* part, int batch, int n_in, int n_blocks, int groups, int hq,
                                float* scores, cudaStream_t stream);
int score_smem_bytes(int mode, int head_dim);

// prefill attention of the window and lookahead rows (attn.cu)
struct AttnParams {
  int head_dim;
  int n_in;          // input keys per unit
  int n_look;        // lookahead keys per unit
  int rows;          // query rows per unit = g * R, ordered [query head][row]
  int R;             // rows per query head
  uint32_t R_mul;    // ceil(2^32 / R) for R > 1: n / R = umulhi(n, R_mul), exact while n * R < 2^32
  int c0;            // head-local row i sees keys [0, c0 + i) of input + lookahead
  float c2;          // scale * log2(e)
  int row_tiles;     // 128-row Q tiles per unit
  int n_items;       // units * ceil(row_tiles / 2): an item is a pair of Q tiles
  void* out;         // bf16 [units][rows][head_dim]
  float* lse2;       // fp32 [units][rows] or null: log2-domain LSE over the input keys
  uint8_t* off_blocks;   // row offsets for the column pass (row_tiles blocks per unit) or null
};
// maps: q [units][rows][d], k and v [units][n_in][d], lookahead k and v [units][n_look][d]
cudaError_t launch_attn(int head_dim, const CUtensorMap (&maps)[5], const AttnParams& p, int grid,
                        cudaStream_t stream);

// Vertical-Slash sparse prefill attention (vs.cu)
constexpr int kVsMaxN = 65536;      // keys per unit (the pattern's bitmaps live in shared memory)
constexpr int kVsMaxVert = 4096;    // vertical columns per unit
struct VsParams {
  int n;             // keys per unit
  int n_q;           // query rows per head: positions n - n_q .. n - 1
  int g;             // query heads per unit
  int n_v, n_s;      // vertical columns and slash offsets per unit
  float c2;          // scale * log2(e)
  int row_blocks;    // ceil(n_q / 128)
  int n_items;       // units * ceil(g / 2) * row_blocks: an item is a pair of query heads
  const int* vert;   // [units][n_v] ascending key indices
  const int* slash;  // [units][n_s] ascending offsets
  void* out;         // bf16 [units * g][n_q][d]
  float* lse2;       // fp32 [units * g][n_q] or null
};
// maps: q [units*g][n_q][d], k and v [units][n][d], gathered vertical k and v [units][n_v][d]
cudaError_t launch_vs_attn(int head_dim, const CUtensorMap (&maps)[5], const VsParams& p, int grid,
                           cudaStream_t stream);

// pooling + top-k selection (select.cu)
enum PoolMode : int {
  POOL_MAX = 0,   // max over the clipped window
  POOL_AVG = 1,   // sum over the clipped window / its length
};
cudaError_t launch_topk(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                        int n_tail, int* idx, float* pooled, void* ws, cudaStream_t stream);
size_t topk_ws_bytes(int units, int n_cand);

// row gather (compact.cu)
cudaError_t launch_compact(const void* k, const void* v, int units, int n_src, int row_bytes, const int* idx,
                           int n_idx, int units_per_idx, void* k_out, void* v_out, cudaStream_t stream);

}  // namespace spk
