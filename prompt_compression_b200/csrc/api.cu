// api.cu -- the extern "C" boundary declared in include/speckv.h.
//
// Host side only: validates arguments (before any launch), builds the TMA
// tensor maps, picks the persistent grid and enqueues the kernels on the
// caller's stream.  No allocation, no host synchronisation on the compute
// paths.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/speckv.h"
#include "common.cuh"
#include "exp2_poly.cuh"
#include "score.cuh"

namespace spk {
SPK_ERROR_READER(device_errors_api)

// decode.cu
cudaError_t launch_decode(const void* q, const void* k, const void* v, float* out, int units, int g,
                          int head_dim, int n_kv, float c2, cudaStream_t stream);

namespace {

thread_local char g_msg[512] = "";

spk_status fail(spk_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return st;
}

spk_status ok() {
  g_msg[0] = 0;
  return SPK_OK;
}

spk_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SPK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  return sms;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 view [n_units][n_rows][head_dim] read in 128-row x 64-column
// boxes with the 128-byte swizzle the UMMA descriptors expect; rows past
// n_rows read as zero.
spk_status make_map(CUtensorMap* map, const void* base, int head_dim, long long n_rows, long long n_units) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(SPK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(n_rows),
                              static_cast<cuuint64_t>(n_units)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(n_rows) * head_dim * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SPK_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return SPK_OK;
}

struct SpeckvGeom {
  long long units, rows, n_pre;
  int g, R;
};

spk_status check_speckv(const spk_speckv_shape* s, SpeckvGeom& g) {
  if (s == nullptr) return fail(SPK_ERR_ARG, "shape is NULL");
  if (s->batch < 1 || s->layers < 1 || s->hq < 1 || s->hkv < 1 || s->n_in < 1)
    return fail(SPK_ERR_ARG, "batch, layers, hq, hkv and n_in must be >= 1");
  if (s->hq % s->hkv != 0) return fail(SPK_ERR_ARG, "hq (%d) must be a multiple of hkv (%d)", s->hq, s->hkv);
  if (s->n_window < 0 || s->n_lookahead < 0 || s->n_window > s->n_in)
    return fail(SPK_ERR_ARG, "need 0 <= n_window <= n_in and n_lookahead >= 0");
  if (s->n_window + s->n_lookahead < 1) return fail(SPK_ERR_ARG, "n_window + n_lookahead must be >= 1");
  if (!(s->scale > 0.f) || !std::isfinite(s->scale)) return fail(SPK_ERR_ARG, "scale must be finite and > 0");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(SPK_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  g.g = s->hq / s->hkv;
  g.R = s->n_window + s->n_lookahead;
  g.rows = static_cast<long long>(g.g) * g.R;
  if (g.rows > kRowsMax)
    return fail(SPK_ERR_UNSUPPORTED, "(hq/hkv) * (n_window + n_lookahead) = %lld exceeds %d", g.rows, kRowsMax);
  g.units = static_cast<long long>(s->batch) * s->layers * s->hkv;
  if (g.units * ((s->n_in + 255) / 256) > 0x7fffffffLL || g.units * 8 > 0x7fffffffLL)
    return fail(SPK_ERR_UNSUPPORTED, "too many units");
  g.n_pre = s->n_in - s->n_window;
  return SPK_OK;
}

ScoreParams base_params(int head_dim, int n_in, const SpeckvGeom& g, int c0, float scale, int hkv,
                        int layers_used, int layers_total, int l_skip) {
  ScoreParams p;
  memset(&p, 0, sizeof p);
  p.head_dim = head_dim;
  p.n_in = n_in;
  p.rows = static_cast<int>(g.rows);
  p.R = g.R;
  p.R_mul = g.R > 1 ? static_cast<uint32_t>(((1ull << 32) + g.R - 1) / g.R) : 0u;
  p.c0 = c0;
  p.c2 = scale * 1.4426950408889634f;
  p.hkv = hkv;
  p.layers_used = layers_used;
  p.layers_total = layers_total;
  p.l_skip = l_skip;
  p.n_units = static_cast<int>(g.units);
  return p;
}

spk_status run_lse(ScoreParams p, const CUtensorMap& qmap, const CUtensorMap& kmap, int head_dim,
                   cudaStream_t stream) {
  p.n_blocks = (p.rows + 255) / 256;
  p.n_items = p.n_units * p.n_blocks;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_score(MODE_LSE, head_dim, qmap, kmap, p, grid, stream);
  if (e != cudaSuccess) return cuda_fail(e, "row-LSE launch");
  return SPK_OK;
}

}  // namespace
}  // namespace spk

using namespace spk;

extern "C" {

const char* spk_last_error(void) { return g_msg; }

// Row offsets between the passes: one kOffBlockBytes block (32 bytes per row)
// per 128-row tile of each unit.
static long long row_tiles(long long rows) { return (rows + 127) / 128; }
static size_t offset_bytes(long long units, long long rows) {
  return static_cast<size_t>(units) * static_cast<size_t>(row_tiles(rows)) * kOffBlockBytes;
}

size_t speckv_workspace_size(const spk_speckv_shape* s) {
  SpeckvGeom g;
  if (check_speckv(s, g) != SPK_OK) return 0;
  return round_up(offset_bytes(g.units, g.rows), 256);
}

static spk_status speckv_maps(const spk_speckv_shape* s, const void* q, const void* k, const SpeckvGeom& g,
                              CUtensorMap* qmap, CUtensorMap* kmap) {
  if (q == nullptr || k == nullptr) return fail(SPK_ERR_ARG, "q and k must be non-NULL device pointers");
  if (!aligned16(q) || !aligned16(k)) return fail(SPK_ERR_ARG, "q and k must be 16-byte aligned");
  spk_status st = make_map(qmap, q, s->head_dim, g.rows, g.units);
  if (st != SPK_OK) return st;
  return make_map(kmap, k, s->head_dim, s->n_in, g.units);
}

spk_status speckv_row_lse(const spk_speckv_shape* s, const void* q, const void* k, float* lse2, void* stream) {
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  if (lse2 == nullptr) return fail(SPK_ERR_ARG, "lse2 must be non-NULL");
  CUtensorMap qmap, kmap;
  if ((st = speckv_maps(s, q, k, g, &qmap, &kmap)) != SPK_OK) return st;
  ScoreParams p = base_params(s->head_dim, s->n_in, g, s->n_in - s->n_window + 1, s->scale, s->hkv, s->layers,
                              s->layers, 0);
  p.lse2 = lse2;
  p.lse_stride = static_cast<int>(g.rows);
  st = run_lse(p, qmap, kmap, s->head_dim, static_cast<cudaStream_t>(stream));
  return st == SPK_OK ? ok() : st;
}

// Pass 1 into the workspace: every query row's offset -lse2/c2 as the
// operand blocks of pass 2's extra UMMA K-step.
spk_status speckv_row_offsets(const spk_speckv_shape* s, const void* q, const void* k, void* ws, size_t ws_bytes,
                              void* stream) {
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  const size_t need = speckv_workspace_size(s);
  if (ws == nullptr || ws_bytes < need)
    return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  CUtensorMap qmap, kmap;
  if ((st = speckv_maps(s, q, k, g, &qmap, &kmap)) != SPK_OK) return st;
  ScoreParams p = base_params(s->head_dim, s->n_in, g, s->n_in - s->n_window + 1, s->scale, s->hkv, s->layers,
                              s->layers, 0);
  p.off_blocks = static_cast<uint8_t*>(ws);
  p.off_tiles = static_cast<int>(row_tiles(g.rows));
  st = run_lse(p, qmap, kmap, s->head_dim, static_cast<cudaStream_t>(stream));
  return st == SPK_OK ? ok() : st;
}

// Pass 2 from a workspace that speckv_row_offsets filled for the same shape, q and k.
spk_status speckv_colsum(const spk_speckv_shape* s, const void* q, const void* k, float* scores, float* window_mass,
                         const void* ws, size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  if (g.n_pre > 0 && scores == nullptr) return fail(SPK_ERR_ARG, "scores must be non-NULL when n_window < n_in");
  const size_t need = speckv_workspace_size(s);
  if (ws == nullptr || ws_bytes < need)
    return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  const int n_cols = static_cast<int>(window_mass ? s->n_in : g.n_pre);
  if (n_cols == 0) return ok();
  CUtensorMap qmap, kmap;
  if ((st = speckv_maps(s, q, k, g, &qmap, &kmap)) != SPK_OK) return st;
  ScoreParams p = base_params(s->head_dim, s->n_in, g, s->n_in - s->n_window + 1, s->scale, s->hkv, s->layers,
                              s->layers, 0);
  p.off_blocks = static_cast<uint8_t*>(const_cast<void*>(ws));
  p.off_tiles = static_cast<int>(row_tiles(g.rows));
  p.n_pre = static_cast<int>(g.n_pre);
  p.n_cols = n_cols;
  p.out0 = scores;
  p.out1 = window_mass;
  p.n_blocks = (n_cols + 255) / 256;
  p.n_items = p.n_units * p.n_blocks;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_score(MODE_COLSUM, s->head_dim, kmap, qmap, p, grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "column-sum launch");
  return ok();
}

spk_status speckv_score(const spk_speckv_shape* s, const void* q, const void* k, float* scores,
                        float* window_mass, void* ws, size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  if (g.n_pre > 0 && scores == nullptr) return fail(SPK_ERR_ARG, "scores must be non-NULL when n_window < n_in");
  const size_t need = speckv_workspace_size(s);
  if (ws == nullptr || ws_bytes < need)
    return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  if ((window_mass ? s->n_in : g.n_pre) == 0) return ok();
  if ((st = speckv_row_offsets(s, q, k, ws, ws_bytes, stream)) != SPK_OK) return st;
  return speckv_colsum(s, q, k, scores, window_mass, ws, ws_bytes, stream);
}

// Prefill attention of the window and lookahead rows (attn.cu): outputs, the
// input-key LSE and, when a workspace is given, the column pass's row offsets.
spk_status speckv_prefill_attention(const spk_speckv_shape* s, const void* q, const void* k, const void* v,
                                   const void* k_look, const void* v_look, void* out, float* lse2, void* ws,
                                   size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return fail(SPK_ERR_ARG, "q, k, v and out must be non-NULL device pointers");
  if (s->n_lookahead > 0 && (k_look == nullptr || v_look == nullptr))
    return fail(SPK_ERR_ARG, "k_look and v_look must be non-NULL when n_lookahead > 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (s->n_lookahead > 0 && (!aligned16(k_look) || !aligned16(v_look))))
    return fail(SPK_ERR_ARG, "q, k, v, k_look, v_look and out must be 16-byte aligned");
  if (ws != nullptr) {
    const size_t need = speckv_workspace_size(s);
    if (ws_bytes < need) return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  }
  const long long tiles = row_tiles(g.rows);
  if (g.units * tiles > 0x7fffffffLL) return fail(SPK_ERR_UNSUPPORTED, "too many units");
  CUtensorMap maps[5];
  if ((st = make_map(&maps[0], q, s->head_dim, g.rows, g.units)) != SPK_OK) return st;
  if ((st = make_map(&maps[1], k, s->head_dim, s->n_in, g.units)) != SPK_OK) return st;
  if ((st = make_map(&maps[2], v, s->head_dim, s->n_in, g.units)) != SPK_OK) return st;
  if (s->n_lookahead > 0) {
    if ((st = make_map(&maps[3], k_look, s->head_dim, s->n_lookahead, g.units)) != SPK_OK) return st;
    if ((st = make_map(&maps[4], v_look, s->head_dim, s->n_lookahead, g.units)) != SPK_OK) return st;
  } else {
    maps[3] = maps[1];   // never read: no lookahead tiles
    maps[4] = maps[2];
  }
  AttnParams p;
  memset(&p, 0, sizeof p);
  p.head_dim = s->head_dim;
  p.n_in = s->n_in;
  p.n_look = s->n_lookahead;
  p.rows = static_cast<int>(g.rows);
  p.R = g.R;
  p.c0 = s->n_in - s->n_window + 1;
  p.c2 = s->scale * 1.4426950408889634f;
  p.row_tiles = static_cast<int>(tiles);
  p.n_items = static_cast<int>(g.units * ((tiles + 1) / 2));   // pairs of Q tiles
  p.out = out;
  p.lse2 = lse2;
  p.off_blocks = static_cast<uint8_t*>(ws);
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_attn(s->head_dim, maps, p, grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
  return ok();
}

// ------------------------------------------------------------------ Vertical-Slash sparse prefill
static spk_status check_vs(const spk_vs_shape* s, long long& units) {
  if (s == nullptr) return fail(SPK_ERR_ARG, "shape is NULL");
  if (s->batch < 1 || s->layers < 1 || s->hq < 1 || s->hkv < 1 || s->n < 1 || s->n_q < 1)
    return fail(SPK_ERR_ARG, "batch, layers, hq, hkv, n and n_q must be >= 1");
  if (s->hq % s->hkv != 0) return fail(SPK_ERR_ARG, "hq (%d) must be a multiple of hkv (%d)", s->hq, s->hkv);
  if (s->n_q > s->n) return fail(SPK_ERR_ARG, "n_q must be <= n");
  if (s->n_vertical < 0 || s->n_slash < 0) return fail(SPK_ERR_ARG, "n_vertical and n_slash must be >= 0");
  if (!(s->scale > 0.f) || !std::isfinite(s->scale)) return fail(SPK_ERR_ARG, "scale must be finite and > 0");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(SPK_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  if (s->n > kVsMaxN) return fail(SPK_ERR_UNSUPPORTED, "n = %d exceeds %d", s->n, kVsMaxN);
  if (s->n_vertical > kVsMaxVert) return fail(SPK_ERR_UNSUPPORTED, "n_vertical = %d exceeds %d", s->n_vertical, kVsMaxVert);
  if (s->n_slash > s->n) return fail(SPK_ERR_ARG, "n_slash must be <= n");
  units = static_cast<long long>(s->batch) * s->layers * s->hkv;
  const long long items = units * (s->hq / s->hkv) * ((s->n_q + 127) / 128);
  if (items > 0x7fffffffLL || units * (s->hq / s->hkv) > 0x7fffffffLL) return fail(SPK_ERR_UNSUPPORTED, "too many units");
  return SPK_OK;
}

size_t vs_workspace_size(const spk_vs_shape* s) {
  long long units;
  if (check_vs(s, units) != SPK_OK) return 0;
  return round_up(2 * static_cast<size_t>(units) * s->n_vertical * s->head_dim * 2, 256);
}

spk_status vs_sparse_attention(const spk_vs_shape* s, const void* q, const void* k, const void* v,
                               const int32_t* vertical, const int32_t* slash, void* out, float* lse2, void* ws,
                               size_t ws_bytes, void* stream) {
  long long units;
  spk_status st = check_vs(s, units);
  if (st != SPK_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return fail(SPK_ERR_ARG, "q, k, v and out must be non-NULL device pointers");
  if ((s->n_vertical > 0 && vertical == nullptr) || (s->n_slash > 0 && slash == nullptr))
    return fail(SPK_ERR_ARG, "vertical / slash must be non-NULL when their counts are > 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SPK_ERR_ARG, "q, k, v and out must be 16-byte aligned");
  const size_t need = vs_workspace_size(s);
  if (s->n_vertical > 0) {
    if (ws == nullptr || ws_bytes < need)
      return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
    if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  }
  const int g = s->hq / s->hkv;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* kvert = static_cast<uint8_t*>(ws);
  uint8_t* vvert = kvert + static_cast<size_t>(units) * s->n_vertical * s->head_dim * 2;
  CUtensorMap maps[5];
  if ((st = make_map(&maps[0], q, s->head_dim, s->n_q, units * g)) != SPK_OK) return st;
  if ((st = make_map(&maps[1], k, s->head_dim, s->n, units)) != SPK_OK) return st;
  if ((st = make_map(&maps[2], v, s->head_dim, s->n, units)) != SPK_OK) return st;
  if (s->n_vertical > 0) {
    if ((st = make_map(&maps[3], kvert, s->head_dim, s->n_vertical, units)) != SPK_OK) return st;
    if ((st = make_map(&maps[4], vvert, s->head_dim, s->n_vertical, units)) != SPK_OK) return st;
    // the vertical keys' K and V rows, gathered once per unit (indices checked on the device)
    cudaError_t e = launch_compact(k, v, static_cast<int>(units), s->n, s->head_dim * 2, vertical, s->n_vertical, 1,
                                   kvert, vvert, cs);
    if (e != cudaSuccess) return cuda_fail(e, "vertical gather launch");
  } else {
    maps[3] = maps[1];   // never read: no vertical tiles
    maps[4] = maps[2];
  }
  VsParams p;
  memset(&p, 0, sizeof p);
  p.n = s->n;
  p.n_q = s->n_q;
  p.g = g;
  p.n_v = s->n_vertical;
  p.n_s = s->n_slash;
  p.c2 = s->scale * 1.4426950408889634f;
  p.row_blocks = (s->n_q + 127) / 128;
  p.n_items = static_cast<int>(units * ((g + 1) / 2) * p.row_blocks);   // pairs of query heads
  p.vert = vertical;
  p.slash = slash;
  p.out = out;
  p.lse2 = lse2;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_vs_attn(s->head_dim, maps, p, grid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "Vertical-Slash attention launch");
  return ok();
}

// ------------------------------------------------------------------ SpecPC
static spk_status check_specpc(const spk_specpc_shape* s, SpeckvGeom& g) {
  if (s == nullptr) return fail(SPK_ERR_ARG, "shape is NULL");
  if (s->batch < 1 || s->layers < 1 || s->hq < 1 || s->hkv < 1 || s->n_in < 1 || s->n_rows < 1)
    return fail(SPK_ERR_ARG, "batch, layers, hq, hkv, n_in and n_rows must be >= 1");
  if (s->hq % s->hkv != 0) return fail(SPK_ERR_ARG, "hq (%d) must be a multiple of hkv (%d)", s->hq, s->hkv);
  if (s->l_skip < 0 || s->l_skip >= s->layers) return fail(SPK_ERR_ARG, "need 0 <= l_skip < layers");
  if (s->n_lookahead < 1) return fail(SPK_ERR_ARG, "n_lookahead must be >= 1");
  if (static_cast<long long>(s->n_rows) > static_cast<long long>(s->n_in) + s->n_lookahead - 1)
    return fail(SPK_ERR_ARG, "n_rows must be <= n_in + n_lookahead - 1");
  if (!(s->scale > 0.f) || !std::isfinite(s->scale)) return fail(SPK_ERR_ARG, "scale must be finite and > 0");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(SPK_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  g.g = s->hq / s->hkv;
  if (s->hq > kHeadsMax) return fail(SPK_ERR_UNSUPPORTED, "hq = %d exceeds %d", s->hq, kHeadsMax);
  g.R = s->n_rows;
  g.rows = static_cast<long long>(g.g) * g.R;
  if (g.rows > kRowsMax)
    return fail(SPK_ERR_UNSUPPORTED, "(hq/hkv) * n_rows = %lld exceeds %d", g.rows, kRowsMax);
  g.units = static_cast<long long>(s->batch) * (s->layers - s->l_skip) * s->hkv;
  if (static_cast<long long>(s->batch) * s->layers * s->hkv * 8 > 0x7fffffffLL)
    return fail(SPK_ERR_UNSUPPORTED, "too many units");
  g.n_pre = s->n_in;
  return SPK_OK;
}

// SpecPC column pass: items are (batch element, 256-key block) pairs; when
// they would leave SMs idle, each block's (KV head, layer) segments are split
// into `groups` contiguous groups, one item each, whose per-head partial sums
// a merge kernel adds in a fixed order.  groups is the smallest count, up to
// 16 and to the number of segments, that fills the grid's waves to >= 95 %
// (else the best fill found).
static int specpc_groups(long long items, int nseg, int sms) {
  auto fill = [&](int gcount) {
    const long long n = items * gcount;
    const long long waves = (n + sms - 1) / sms;
    return static_cast<double>(n) / static_cast<double>(waves * sms);
  };
  int best = 1;
  double best_fill = fill(1);
  for (int gcount = 1; gcount <= 16 && gcount <= nseg; ++gcount) {
    const double f = fill(gcount);
    if (f >= 0.95) return gcount;
    if (f > best_fill + 1e-9) { best = gcount; best_fill = f; }
  }
  return best;
}

struct SpecpcPlan {
  int n_blocks, groups;
  size_t off_bytes, part_bytes;
};

static SpecpcPlan specpc_plan(const spk_specpc_shape* s, const SpeckvGeom& g) {
  SpecpcPlan pl;
  pl.n_blocks = (s->n_in + 255) / 256;
  pl.groups = specpc_groups(static_cast<long long>(s->batch) * pl.n_blocks, s->hkv * (s->layers - s->l_skip),
                            num_sms());
  pl.off_bytes = round_up(offset_bytes(g.units, g.rows), 256);
  pl.part_bytes = pl.groups > 1 ? static_cast<size_t>(s->batch) * pl.n_blocks * pl.groups * s->hq * 256 * 4 : 0;
  return pl;
}

size_t specpc_workspace_size(const spk_specpc_shape* s) {
  SpeckvGeom g;
  if (check_specpc(s, g) != SPK_OK) return 0;
  const SpecpcPlan pl = specpc_plan(s, g);
  return pl.off_bytes + round_up(pl.part_bytes, 256);
}

static spk_status specpc_prepare(const spk_specpc_shape* s, const void* q, const void* k, const void* ws,
                                 size_t ws_bytes, SpeckvGeom& g, CUtensorMap* qmap, CUtensorMap* kmap, ScoreParams& p) {
  spk_status st = check_specpc(s, g);
  if (st != SPK_OK) return st;
  if (q == nullptr || k == nullptr) return fail(SPK_ERR_ARG, "q and k must be non-NULL device pointers");
  if (!aligned16(q) || !aligned16(k)) return fail(SPK_ERR_ARG, "q and k must be 16-byte aligned");
  const size_t need = specpc_workspace_size(s);
  if (ws == nullptr || ws_bytes < need)
    return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (!aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  const long long all_units = static_cast<long long>(s->batch) * s->layers * s->hkv;
  if ((st = make_map(qmap, q, s->head_dim, g.rows, all_units)) != SPK_OK) return st;
  if ((st = make_map(kmap, k, s->head_dim, s->n_in, all_units)) != SPK_OK) return st;
  const int c0 = s->n_in + s->n_lookahead - s->n_rows;
  p = base_params(s->head_dim, s->n_in, g, c0, s->scale, s->hkv, s->layers - s->l_skip, s->layers, s->l_skip);
  p.off_blocks = static_cast<uint8_t*>(const_cast<void*>(ws));
  p.off_tiles = static_cast<int>(row_tiles(g.rows));
  p.seg_groups = 1;
  return SPK_OK;
}

spk_status specpc_row_offsets(const spk_specpc_shape* s, const void* q, const void* k, const float* w, void* ws,
                              size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  CUtensorMap qmap, kmap;
  ScoreParams p;
  spk_status st = specpc_prepare(s, q, k, ws, ws_bytes, g, &qmap, &kmap, p);
  if (st != SPK_OK) return st;
  if (w == nullptr) return fail(SPK_ERR_ARG, "row_weights must be a non-NULL device pointer");
  p.row_weights = w;
  st = run_lse(p, qmap, kmap, s->head_dim, static_cast<cudaStream_t>(stream));
  return st == SPK_OK ? ok() : st;
}

spk_status specpc_colsum(const spk_specpc_shape* s, const void* q, const void* k, float* scores, void* ws,
                         size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  CUtensorMap qmap, kmap;
  ScoreParams p;
  spk_status st = specpc_prepare(s, q, k, ws, ws_bytes, g, &qmap, &kmap, p);
  if (st != SPK_OK) return st;
  if (scores == nullptr) return fail(SPK_ERR_ARG, "scores must be a non-NULL device pointer");
  const SpecpcPlan pl = specpc_plan(s, g);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  p.n_pre = s->n_in;
  p.n_cols = s->n_in;
  p.out0 = scores;
  p.n_blocks = pl.n_blocks;
  p.seg_groups = pl.groups;
  p.part = pl.groups > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_bytes) : nullptr;
  p.n_items = s->batch * pl.n_blocks * pl.groups;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_score(MODE_COLSUM_PC, s->head_dim, kmap, qmap, p, grid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "SpecPC column-sum launch");
  if (pl.groups > 1) {
    e = launch_specpc_merge(p.part, s->batch, s->n_in, pl.n_blocks, pl.groups, s->hq, scores, cs);
    if (e != cudaSuccess) return cuda_fail(e, "SpecPC merge launch");
  }
  return ok();
}

spk_status specpc_score(const spk_specpc_shape* s, const void* q, const void* k, const float* w, float* scores,
                        void* ws, size_t ws_bytes, void* stream) {
  SpeckvGeom g;
  spk_status st = check_specpc(s, g);
  if (st != SPK_OK) return st;
  if (q == nullptr || k == nullptr || w == nullptr || scores == nullptr)
    return fail(SPK_ERR_ARG, "q, k, row_weights and scores must be non-NULL device pointers");
  if ((st = specpc_row_offsets(s, q, k, w, ws, ws_bytes, stream)) != SPK_OK) return st;
  return specpc_colsum(s, q, k, scores, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ selection
size_t topk_workspace_size(int units, int n_cand) {
  if (units < 0 || n_cand < 0) return 0;
  return round_up(topk_ws_bytes(units, n_cand), 256);
}

static spk_status topk_common(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                              int n_tail, int32_t* idx, float* pooled, void* ws, size_t ws_bytes, void* stream) {
  if (units < 0 || n_cand < 0 || k < 0 || n_tail < 0) return fail(SPK_ERR_ARG, "negative size");
  if (pool_kernel < 1 || (pool_kernel & 1) == 0) return fail(SPK_ERR_ARG, "pool_kernel must be odd and >= 1");
  if (pool_mode != SPK_POOL_MAX && pool_mode != SPK_POOL_AVG)
    return fail(SPK_ERR_ARG, "pool_mode must be SPK_POOL_MAX (0) or SPK_POOL_AVG (1), got %d", pool_mode);
  if (units == 0) return ok();
  const long long out_len = static_cast<long long>(k < n_cand ? k : n_cand) + n_tail;
  if (out_len > 0 && idx == nullptr) return fail(SPK_ERR_ARG, "idx must be non-NULL");
  if (n_cand > 0 && scores == nullptr) return fail(SPK_ERR_ARG, "scores must be non-NULL");
  const size_t need = topk_workspace_size(units, n_cand);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(SPK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (need > 0 && !aligned16(ws)) return fail(SPK_ERR_ARG, "workspace must be 16-byte aligned");
  if (static_cast<long long>(units) > 0x7fffffffLL / (out_len > 0 ? out_len : 1) && out_len > 0)
    return fail(SPK_ERR_UNSUPPORTED, "output too large");
  cudaError_t e = launch_topk(scores, units, n_cand, pool_mode, pool_kernel, k, n_tail, idx, pooled, ws,
                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  return ok();
}

spk_status topk_select(const float* scores, int units, int n_cand, int pool_kernel, int k, int n_tail,
                       int32_t* idx, float* pooled, void* ws, size_t ws_bytes, void* stream) {
  return topk_common(scores, units, n_cand, SPK_POOL_MAX, pool_kernel, k, n_tail, idx, pooled, ws, ws_bytes, stream);
}

spk_status topk_select_pool(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                            int n_tail, int32_t* idx, float* pooled, void* ws, size_t ws_bytes, void* stream) {
  return topk_common(scores, units, n_cand, pool_mode, pool_kernel, k, n_tail, idx, pooled, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ compaction
spk_status kv_compact(const void* k, const void* v, int units, int n_src, int head_dim, int elem_bytes,
                      const int32_t* idx, int n_idx, int units_per_idx, void* k_out, void* v_out, void* stream) {
  if (units < 0 || n_src < 0 || n_idx < 0 || head_dim < 1 || elem_bytes < 1 || units_per_idx < 1)
    return fail(SPK_ERR_ARG, "invalid sizes");
  if (units % units_per_idx != 0) return fail(SPK_ERR_ARG, "units must be a multiple of units_per_idx");
  const long long row_bytes = static_cast<long long>(head_dim) * elem_bytes;
  if (row_bytes % 16 != 0) return fail(SPK_ERR_UNSUPPORTED, "head_dim * elem_bytes must be a multiple of 16");
  if (units == 0 || n_idx == 0) return ok();
  if (k == nullptr || k_out == nullptr || idx == nullptr) return fail(SPK_ERR_ARG, "k, k_out, idx must be non-NULL");
  if ((v == nullptr) != (v_out == nullptr)) return fail(SPK_ERR_ARG, "v and v_out must both be set or both NULL");
  if (!aligned16(k) || !aligned16(k_out) || (v && (!aligned16(v) || !aligned16(v_out))))
    return fail(SPK_ERR_ARG, "k, v, k_out, v_out must be 16-byte aligned");
  cudaError_t e = launch_compact(k, v, units, n_src, static_cast<int>(row_bytes), idx, n_idx, units_per_idx, k_out,
                                 v_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "compaction launch");
  return ok();
}

// ------------------------------------------------------------------ device errors
// ------------------------------------------------------------------ decode
spk_status decode_attention(int batch, int layers, int hq, int hkv, int head_dim, int n_kv, float scale,
                            const void* q, const void* k, const void* v, float* out, void* stream) {
  if (batch < 1 || layers < 1 || hq < 1 || hkv < 1 || n_kv < 1)
    return fail(SPK_ERR_ARG, "batch, layers, hq, hkv and n_kv must be >= 1");
  if (hq % hkv != 0) return fail(SPK_ERR_ARG, "hq (%d) must be a multiple of hkv (%d)", hq, hkv);
  if (hq / hkv > 8) return fail(SPK_ERR_UNSUPPORTED, "hq / hkv = %d exceeds 8", hq / hkv);
  if (head_dim != 64 && head_dim != 128)
    return fail(SPK_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(SPK_ERR_ARG, "scale must be finite and > 0");
  const long long units = static_cast<long long>(batch) * layers * hkv;
  if (units > 0x7fffffffLL || static_cast<long long>(n_kv) * head_dim > (1LL << 40) / units)
    return fail(SPK_ERR_UNSUPPORTED, "too many units or rows");
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return fail(SPK_ERR_ARG, "q, k, v and out must be non-NULL device pointers");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SPK_ERR_ARG, "q, k, v and out must be 16-byte aligned");
  cudaError_t e = launch_decode(q, k, v, out, static_cast<int>(units), hq / hkv, head_dim, n_kv,
                                scale * 1.4426950408889634f, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  return ok();
}

spk_status spk_mapped_host_pointer(const void* host, void** dev) {
  if (host == nullptr || dev == nullptr) return fail(SPK_ERR_ARG, "host and dev must be non-NULL");
  void* d = nullptr;
  cudaError_t e = cudaHostGetDevicePointer(&d, const_cast<void*>(host), 0);
  if (e != cudaSuccess) {
    cudaGetLastError();   // not sticky: clear it
    return cuda_fail(e, "host memory is not page-locked and mapped into the device");
  }
  *dev = d;
  return ok();
}

spk_status spk_device_error(int* status, int* site, int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  // every translation unit's error word, the first set one in this order
  // reported (the others are cleared with it)
  cudaError_t (*const readers[])(int*, int*, bool) = {device_errors_api, device_errors_score, device_errors_attn,
                                                       device_errors_vs, device_errors_compact};
  int code = 0, where = 0;
  for (auto rd : readers) {
    int c = 0, w = 0;
    if ((e = rd(&c, &w, clear != 0)) != cudaSuccess) return cuda_fail(e, "reading a device error word");
    if (code == 0 && c != 0) {
      code = c;
      where = w;
    }
  }
  if (status) *status = code == SPK_DEVERR_NONE ? SPK_OK : (code == SPK_DEVERR_TIMEOUT ? SPK_ERR_TIMEOUT : SPK_ERR_ARG);
  if (site) *site = where;
  return ok();
}

}  // extern "C"

namespace spk {
namespace {
// One thread waits on a barrier that nothing will ever complete; the bounded
// wait gives up after limit_ns, records the timeout and returns.
__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), 999, limit_ns);
  }
}
}  // namespace
}  // namespace spk

extern "C" spk_status spk_selftest_wait_timeout(long long limit_ns, void* stream) {
  if (limit_ns < 1000) limit_ns = 1000;
  if (limit_ns > 1000000000LL) limit_ns = 1000000000LL;
  spk::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return spk::cuda_fail(e, "self-test launch");
  return spk::ok();
}

// ---------------------------------------------------------------------------
// speckv_score_static_ws: speckv_score without a caller-provided workspace.
//
// Some callers cannot allocate device memory on this path: serving engines
// that reserve nearly all of HBM up front for their KV-cache pool and hand
// memory out only through their own allocator, and plugin hosts that give a
// plugin no access to the CUDA allocator.  They also cannot always find room
// for a workspace.  This entry point keeps the row offsets that pass 1 hands
// to pass 2 in a fixed array that lives in the library image itself, so a
// call allocates nothing (no cudaMalloc, no cudaFree, no allocating library
// routine).
//
// Limits and behaviour:
//   - the scratch holds kStaticOffBytes = 16 MiB, 32 bytes per query row with
//     each unit's rows rounded up to 128: 524,288 rows (one batch element of
//     a 64-layer, 8-KV-head, 960-row model); a larger shape is rejected with
//     SPK_ERR_UNSUPPORTED before anything is launched;
//   - every GPU that loads the library keeps these 16 MiB until the process exits;
//   - the first call on each device looks up the array's device address with
//     that device current (cudaGetSymbolAddress) and caches it; make that
//     first call before any stream capture;
//   - all calls share the one array and it keeps the previous call's contents.
//     Pass 1 overwrites every entry pass 2 reads, so nothing has to start at
//     zero, but calls whose kernels overlap on the GPU (different streams
//     without ordering between them) race on the array: order them.
// ---------------------------------------------------------------------------
#include <mutex>

namespace spk {
namespace {
constexpr long long kStaticOffBytes = 1LL << 24;
constexpr int kMaxDevices = 64;
static __device__ __align__(256) uint8_t g_static_off[kStaticOffBytes];
uint8_t* g_static_off_addr[kMaxDevices] = {};
std::mutex g_static_off_mu;

// Device address of g_static_off on the current device (looked up once per device).
spk_status static_off_address(uint8_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SPK_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_static_off_mu);
  if (g_static_off_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_off);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    g_static_off_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_static_off_addr[dev];
  return SPK_OK;
}
}  // namespace
}  // namespace spk

extern "C" spk_status speckv_score_static_ws(const spk_speckv_shape* s, const void* q, const void* k,
                                             float* scores, float* window_mass, void* stream) {
  using namespace spk;
  SpeckvGeom g;
  spk_status st = check_speckv(s, g);
  if (st != SPK_OK) return st;
  const long long need = static_cast<long long>(offset_bytes(g.units, g.rows));
  if (need > kStaticOffBytes)
    return fail(SPK_ERR_UNSUPPORTED,
                "units * (hq/hkv) * (n_window + n_lookahead) rows, rounded up to 128 per unit, need %lld bytes of "
                "row offsets and exceed the static scratch of %lld bytes; use speckv_score with a workspace",
                need, kStaticOffBytes);
  if (g.n_pre > 0 && scores == nullptr) return fail(SPK_ERR_ARG, "scores must be non-NULL when n_window < n_in");
  const int n_cols = static_cast<int>(window_mass ? s->n_in : g.n_pre);
  if (n_cols == 0) return ok();
  CUtensorMap qmap, kmap;
  if ((st = speckv_maps(s, q, k, g, &qmap, &kmap)) != SPK_OK) return st;
  uint8_t* off = nullptr;
  if ((st = static_off_address(&off)) != SPK_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  ScoreParams p = base_params(s->head_dim, s->n_in, g, s->n_in - s->n_window + 1, s->scale, s->hkv, s->layers,
                              s->layers, 0);
  p.off_blocks = off;
  p.off_tiles = static_cast<int>(row_tiles(g.rows));
  if ((st = run_lse(p, qmap, kmap, s->head_dim, cs)) != SPK_OK) return st;
  p.n_pre = static_cast<int>(g.n_pre);
  p.n_cols = n_cols;
  p.out0 = scores;
  p.out1 = window_mass;
  p.n_blocks = (n_cols + 255) / 256;
  p.n_items = p.n_units * p.n_blocks;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  cudaError_t e = launch_score(MODE_COLSUM, s->head_dim, kmap, qmap, p, grid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "column-sum launch");
  return ok();
}

// ---------------------------------------------------------------------------
// spk_exp2_fma: the FMA-pipe exponential of the scoring epilogues, exposed
// so that tests can compare it with exp2 over its whole argument range.
// ---------------------------------------------------------------------------
namespace spk {
namespace {
__global__ void exp2_fma_kernel(const float* __restrict__ t, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_fma_pair(f2(t[i], t[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_fma_pair(f2(t[i], t[i])).x;
  }
}
}  // namespace
}  // namespace spk

extern "C" spk_status spk_exp2_fma(const float* t, float* y, int n, void* stream) {
  if (n < 0) return spk::fail(SPK_ERR_ARG, "n must be >= 0");
  if (n == 0) return spk::ok();
  if (t == nullptr || y == nullptr) return spk::fail(SPK_ERR_ARG, "t and y must be non-NULL device pointers");
  const int pairs = (n + 1) / 2;
  spk::exp2_fma_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(t, y, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return spk::cuda_fail(e, "exp2 launch");
  return spk::ok();
}
