// K/V cache writer and reader.
//
// The thinker's K/V slice for a unit is written verbatim into the session's
// pre-allocated cache ("Wan-Streamer v0.2" digest, "method overview and
// architecture": each performer rank writes the broadcast slice into its
// pre-sharded local cache).  Unit u goes to ring slot u mod cache_units.
//
// Layout: pool [L][pool_tokens][H * D_h]; a session owns rows
// [base, base + cache_units * T_u + N).  Source slice [L][n_tok][H_src * D_h]:
// a row of the slice may hold more heads than the cache (a rank of a
// head-sharded cache copies its own head range of the broadcast slice).
// Pure HBM copy: one CTA per (layer, token) row of K and V, 16-byte
// streaming loads/stores (the slice is read once and the destination is not
// re-read before it leaves L2).
#include "common.cuh"

namespace sfm {

__global__ void __launch_bounds__(256) kv_append_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ k_pool,
    uint4* __restrict__ v_pool, int n_tok, int unit_tokens, long long pool_tokens, int row_vecs,
    int src_row_vecs, int src_off_vecs, long long base_row, long long first_unit,
    int cache_units) {
  const long long src_row = blockIdx.x;                 // = layer * n_tok + t
  const int layer = (int)(src_row / n_tok);
  const int t = (int)(src_row - (long long)layer * n_tok);
  const int unit = t / unit_tokens;
  const int t_in = t - unit * unit_tokens;
  const long long slot = (first_unit + unit) % cache_units;
  const long long dst_row = (long long)layer * pool_tokens + base_row + slot * unit_tokens + t_in;
  const uint4* ks = k + src_row * src_row_vecs + src_off_vecs;
  const uint4* vs = v + src_row * src_row_vecs + src_off_vecs;
  uint4* kd = k_pool + dst_row * row_vecs;
  uint4* vd = v_pool + dst_row * row_vecs;
  for (int c = threadIdx.x; c < row_vecs; c += blockDim.x) {
    const uint4 a = __ldcs(ks + c);
    const uint4 b = __ldcs(vs + c);
    __stcs(kd + c, a);
    __stcs(vd + c, b);
  }
}

__global__ void __launch_bounds__(256) kv_read_kernel(
    const uint4* __restrict__ k_pool, const uint4* __restrict__ v_pool, uint4* __restrict__ kd,
    uint4* __restrict__ vd, long long src_row0, int row_vecs) {
  const long long r = blockIdx.x;
  const uint4* ks = k_pool + (src_row0 + r) * row_vecs;
  const uint4* vs = v_pool + (src_row0 + r) * row_vecs;
  for (int c = threadIdx.x; c < row_vecs; c += blockDim.x) {
    kd[r * row_vecs + c] = ks[c];
    vd[r * row_vecs + c] = vs[c];
  }
}

static int block_for(int row_vecs) {
  int b = row_vecs < 256 ? row_vecs : 256;
  b = (b + 31) / 32 * 32;
  return b;
}

int launch_kv_append(const void* k, const void* v, void* k_pool, void* v_pool, int n_layers,
                     long long pool_tokens, int row_bytes, int n_tok, int unit_tokens,
                     long long base_row, long long first_unit, int cache_units, cudaStream_t s,
                     int src_row_bytes, int src_off_bytes) {
  const int row_vecs = row_bytes / 16;
  const int src_row_vecs = (src_row_bytes ? src_row_bytes : row_bytes) / 16;
  const long long rows = (long long)n_layers * n_tok;
  if (rows == 0) return SFM_OK;
  kv_append_kernel<<<(unsigned)rows, block_for(row_vecs), 0, s>>>(
      (const uint4*)k, (const uint4*)v, (uint4*)k_pool, (uint4*)v_pool, n_tok, unit_tokens,
      pool_tokens, row_vecs, src_row_vecs, src_off_bytes / 16, base_row, first_unit, cache_units);
  return record_cuda(cudaGetLastError());
}

int launch_kv_read(const void* k_pool, const void* v_pool, void* k_dst, void* v_dst, int layer,
                   long long pool_tokens, int row_bytes, long long row0, long long n_rows,
                   cudaStream_t s) {
  const int row_vecs = row_bytes / 16;
  if (n_rows == 0) return SFM_OK;
  kv_read_kernel<<<(unsigned)n_rows, block_for(row_vecs), 0, s>>>(
      (const uint4*)k_pool, (const uint4*)v_pool, (uint4*)k_dst, (uint4*)v_dst,
      (long long)layer * pool_tokens + row0, row_vecs);
  return record_cuda(cudaGetLastError());
}

}  // namespace sfm
