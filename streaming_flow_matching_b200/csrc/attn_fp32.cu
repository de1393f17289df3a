// Attention of the current unit over [valid cache ; current unit] -- the
// performer form of the block-causal attention of "Wan-Streamer" v0.1 blog
// §3.3: every cached unit precedes the current one and the current unit is
// bidirectional, so every key is visible to every query.  With
// AttnDesc::unit_rows > 0 the general block-causal form: several units of
// queries, each seeing the shared prefix and the units up to its own.
//
//   fp32 mode: one warp per (query row, head) on the CUDA cores.
//   attn_merge_kernel: combines the split-KV partial results of the tcgen05
//   kernel (attn_tc.cu): O = sum_s 2^(lse_s - max) O_s / sum_s 2^(lse_s - max).
#include <math.h>

#include "attn.cuh"

namespace sfm {


// fp32 CUDA-core attention: one warp per (row, head), D a multiple of 32 (<= 128)
__global__ void attn_f32_kernel(AttnDesc a, const float* __restrict__ q,
                                const float* __restrict__ k, const float* __restrict__ v,
                                float* __restrict__ o, int H, int D, float scale_log2,
                                long long total_rows) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= total_rows * H) return;
  const long long row = gw / H;
  const int h = (int)(gw - row * H);
  const int sess = (int)(row / a.rows_per);
  const int ne = D / 32;
  const long long ld = (long long)H * D;
  float qv[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int e = 0; e < ne; ++e) qv[e] = q[row * ld + h * D + lane + 32 * e];
  float m = -INFINITY, l = 0.f;
  const long long kb = a.kbase[sess];
  const int lim = attn_key_limit(a.nkeys[sess], a.rows_per, a.unit_rows,
                                 (int)(row - (long long)sess * a.rows_per));
  for (int t = 0; t < lim; ++t) {
    const float* kr = k + (kb + t) * ld + h * D;
    float s = 0.f;
    for (int e = 0; e < ne; ++e) s = fmaf(qv[e], kr[lane + 32 * e], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    s *= scale_log2;
    const float m_new = fmaxf(m, s);
    const float alpha = exp2f(m - m_new);
    const float p = exp2f(s - m_new);
    l = l * alpha + p;
    const float* vr = v + (kb + t) * ld + h * D;
    for (int e = 0; e < ne; ++e) acc[e] = fmaf(p, vr[lane + 32 * e], acc[e] * alpha);
    m = m_new;
  }
  for (int e = 0; e < ne; ++e) o[row * ld + h * D + lane + 32 * e] = acc[e] / l;
}

// Merge split-KV partials: one warp per (row, head); D = 128 (float4 per lane).
// Every split's log-sum-exp and partial row are loaded up front, so the loads
// of a row are in flight together.  The split count is a template parameter so a
// thread holds exactly its splits' values (a fixed 16-slot version needed 94
// registers and ran at a quarter of the warps an SM can hold).
// The rows of the sessions md lists, each of S partials (one launch per split count).
template <int S>
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         __nv_bfloat16* __restrict__ o,
                                                         long long total_rows, int H, MergeDesc md) {
  const unsigned gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned per = (unsigned)md.rows_per * (unsigned)H;   // (row, head) pairs of a session
  if (gw >= (unsigned)md.n * per) return;
  const unsigned k = gw / per, rh = gw - k * per;
  const unsigned r = rh / (unsigned)H;
  const int h = (int)(rh - r * (unsigned)H);
  const long long row = (long long)md.sess[k] * md.rows_per + r;
  const long long ld = (long long)H * 128;
  float lse[S];
  float4 p[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    lse[s] = __ldcs(lse_part + ((long long)s * total_rows + row) * H + h);
    p[s] = __ldcs(reinterpret_cast<const float4*>(o_part + ((long long)s * total_rows + row) * ld +
                                                  h * 128) + lane);
  }
  float mmax = -INFINITY;
#pragma unroll
  for (int s = 0; s < S; ++s) mmax = fmaxf(mmax, lse[s]);
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < S; ++s) {
    // a split without keys has lse = -inf and weight 0 (its partial row is zeros)
    const float w = lse[s] == -INFINITY ? 0.f : exp2f(lse[s] - mmax);
    wsum += w;
    acc.x = fmaf(w, p[s].x, acc.x);
    acc.y = fmaf(w, p[s].y, acc.y);
    acc.z = fmaf(w, p[s].z, acc.z);
    acc.w = fmaf(w, p[s].w, acc.w);
  }
  const float inv = 1.f / wsum;
  __nv_bfloat16* od = o + row * ld + h * 128 + lane * 4;
  *reinterpret_cast<__nv_bfloat162*>(od) = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  *reinterpret_cast<__nv_bfloat162*>(od + 2) = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
}

template <int S>
static void launch_merge_s(const float* o_part, const float* lse_part, void* o, long long total_rows,
                           int n_heads, int n_splits, const MergeDesc& md, cudaStream_t s) {
  if constexpr (S > 1) {
    if (n_splits != S) {
      launch_merge_s<S - 1>(o_part, lse_part, o, total_rows, n_heads, n_splits, md, s);
      return;
    }
    const long long warps = (long long)md.n * md.rows_per * n_heads;
    attn_merge_kernel<S><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(
        o_part, lse_part, (__nv_bfloat16*)o, total_rows, n_heads, md);
  }
}

size_t attention_workspace_bytes(long long rows, int n_heads, int n_splits) {
  if (n_splits <= 1) return 0;
  return (size_t)n_splits * rows * n_heads * (128 + 1) * sizeof(float);
}

int launch_attention(const AttnDesc& a, const void* q, const void* k, const void* v, void* o,
                     int n_heads, int head_dim, int dtype, int n_splits, float* o_part,
                     float* lse_part, cudaStream_t s) {
  const long long total_rows = (long long)a.n * a.rows_per;
  if (total_rows == 0) return SFM_OK;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)head_dim));
  (void)n_splits;
  (void)o_part;
  (void)lse_part;
  if (dtype == SFM_DTYPE_FP32) {
    ProfScope ps(SFM_PROF_ATTN, s);
    const long long warps = total_rows * n_heads;
    attn_f32_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(
        a, (const float*)q, (const float*)k, (const float*)v, (float*)o, n_heads, head_dim,
        scale_log2, total_rows);
    return record_cuda(cudaGetLastError());
  }
  return SFM_EUNSUPPORTED;   // bf16 attention runs on tcgen05 (attn_tc.cu)
}

int launch_attention_merge(const float* o_part, const float* lse_part, void* o,
                           long long total_rows, int n_heads, int n_splits, const MergeDesc& md,
                           cudaStream_t s) {
  if (n_splits < 2 || n_splits > kMaxSplits || md.rows_per < 1 || md.n < 1 || md.n > kMaxBatch ||
      (long long)md.n * md.rows_per * n_heads * 32 >= (1LL << 31))
    return SFM_EINVAL;
  launch_merge_s<kMaxSplits>(o_part, lse_part, o, total_rows, n_heads, n_splits, md, s);
  return record_cuda(cudaGetLastError());
}

}  // namespace sfm
