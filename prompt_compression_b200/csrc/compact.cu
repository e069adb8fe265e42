// compact.cu -- KV compaction: gather the selected rows of K and V.
//
// "Draft-based Approximate Inference for LLMs" (paper notes), section 关键设计,
// SpecKV: after selection only the chosen KV pairs remain in the cache.
// k_out[u][t] = k[u][idx[u / units_per_idx][t]] (same for v), bytes copied as
// they are.  A row is head_dim * elem_bytes bytes (a multiple of 16); each
// thread moves 16-byte vectors, consecutive threads cover consecutive vectors
// of a row, so a warp reads and writes whole 128..256-byte rows: the gather
// is HBM-bandwidth bound with no re-reads.
#include "common.cuh"
#include "score.cuh"

namespace spk {

SPK_ERROR_READER(device_errors_compact)

namespace {

__global__ void __launch_bounds__(256)
    compact_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, int n_src, int row_vecs,
                   const int* __restrict__ idx, int n_idx, int units_per_idx, uint4* __restrict__ k_out,
                   uint4* __restrict__ v_out, size_t total_vecs) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total_vecs; e += stride) {
    const size_t row = e / row_vecs;                 // output row = u * n_idx + t
    const int vec = static_cast<int>(e - row * row_vecs);
    const size_t u = row / n_idx;
    const int t = static_cast<int>(row - u * n_idx);
    const int src = __ldg(idx + (u / units_per_idx) * n_idx + t);
    if (src < 0 || src >= n_src) {
      if (vec == 0) record_error(SPK_DEVERR_INDEX, static_cast<int>(u));
      continue;
    }
    const size_t s = (u * n_src + src) * row_vecs + vec;
    k_out[e] = __ldcs(k + s);
    if (v != nullptr) v_out[e] = __ldcs(v + s);
  }
}

}  // namespace

cudaError_t launch_compact(const void* k, const void* v, int units, int n_src, int row_bytes, const int* idx,
                           int n_idx, int units_per_idx, void* k_out, void* v_out, cudaStream_t stream) {
  const int row_vecs = row_bytes / 16;
  const size_t total = static_cast<size_t>(units) * n_idx * row_vecs;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  size_t blocks = (total + 255) / 256;
  const size_t cap = static_cast<size_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  compact_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), n_src, row_vecs, idx, n_idx, units_per_idx,
      static_cast<uint4*>(k_out), static_cast<uint4*>(v_out), total);
  return cudaGetLastError();
}

}  // namespace spk
