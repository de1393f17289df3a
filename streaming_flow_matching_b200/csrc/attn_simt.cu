// Attention of the current unit over [valid cache ; current unit] -- the
// performer form of the block-causal attention of "Wan-Streamer" v0.1 blog
// §3.3: every cached unit precedes the current one and the current unit is
// bidirectional, so every key is visible to every query.
//
//   bf16: flash attention on mma.sync m16n8k16 (fp32 accumulate, online
//         softmax in the exp2 domain), 64 query rows x 64 keys per step,
//         cp.async double buffering; the key range can be split across CTAs
//         (split-KV) and merged by attn_merge_kernel.  First, correctness-first
//         path; the tcgen05 kernel replaces it.
//   fp32: one warp per (query row, head), CUDA cores (the fp32 mode).
#include <math.h>

#include "attn.cuh"

namespace sfm {

namespace fa {
constexpr int BQ = 64, BKV = 64, D = 128, THREADS = 128;
constexpr int TILE = BKV * D * 2;                  // 16 KB
constexpr int SMEM = BQ * D * 2 + 4 * TILE;        // Q + 2 x (K, V) = 80 KB

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// [rows][128] bf16 tile, 256-byte rows of 16 chunks, chunk XOR (row & 7)
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * 256 + ((ch ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

// rows [0, n_valid) of a [64][128] tile from g (row stride ld elements), zero-fill beyond
__device__ __forceinline__ void load_rows(uint32_t s, const __nv_bfloat16* g, long long ld,
                                          int n_valid, int tid) {
#pragma unroll
  for (int it = 0; it < (64 * 16) / THREADS; ++it) {
    const int c = tid + it * THREADS;
    const int r = c >> 4, ch = c & 15;
    const bool ok = r < n_valid;
    cp_async16(s + swz(r, ch), g + (ok ? r : 0) * ld + ch * 8, ok);
  }
}

__global__ void __launch_bounds__(THREADS, 2)
    fa_fwd_kernel(AttnDesc a, const __nv_bfloat16* __restrict__ q,
                  const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                  __nv_bfloat16* __restrict__ o, float* __restrict__ o_part,
                  float* __restrict__ lse_part, int H, int n_splits, int qtiles, float scale_log2,
                  long long total_rows) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sess = blockIdx.x / qtiles;
  const int qt = blockIdx.x - sess * qtiles;
  const int h = blockIdx.y, split = blockIdx.z;
  const long long row0 = (long long)sess * a.rows_per + qt * BQ;
  const int q_rows = min(BQ, a.rows_per - qt * BQ);
  const int nkeys = a.nkeys[sess];
  const long long kbase = a.kbase[sess];
  const int ntiles = (nkeys + BKV - 1) / BKV;
  const int tps = (ntiles + n_splits - 1) / n_splits;
  const int t0 = split * tps;
  const int t1 = min(ntiles, t0 + tps);
  const long long ld = (long long)H * D;

  const uint32_t sq = smem_u32(smem);
  const uint32_t sk0 = sq + BQ * D * 2;
  auto sk = [&](int st) { return sk0 + st * 2 * TILE; };
  auto sv = [&](int st) { return sk0 + st * 2 * TILE + TILE; };

  load_rows(sq, q + row0 * ld + h * D, ld, q_rows, tid);
  if (t0 < t1) {
    const int n0 = min(BKV, nkeys - t0 * BKV);
    load_rows(sk(0), k + (kbase + (long long)t0 * BKV) * ld + h * D, ld, n0, tid);
    load_rows(sv(0), v + (kbase + (long long)t0 * BKV) * ld + h * D, ld, n0, tid);
  }
  cp_commit();

  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float acc[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  uint32_t qf[8][4];

  for (int t = t0; t < t1; ++t) {
    const int st = (t - t0) & 1;
    if (t + 1 < t1) {
      const int n1 = min(BKV, nkeys - (t + 1) * BKV);
      load_rows(sk(st ^ 1), k + (kbase + (long long)(t + 1) * BKV) * ld + h * D, ld, n1, tid);
      load_rows(sv(st ^ 1), v + (kbase + (long long)(t + 1) * BKV) * ld + h * D, ld, n1, tid);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (t == t0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldsm_x4(sq + swz(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), qf[kk]);
    }
    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ldsm_x4(sk(st) + swz(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
                b);
        mma16816(s[2 * np], qf[kk], b[0], b[1]);
        mma16816(s[2 * np + 1], qf[kk], b[2], b[3]);
      }
    }
    // scale, mask the ragged last tile, online softmax (rows g and g + 8)
    const int kvalid = nkeys - t * BKV;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 8 + (lane & 3) * 2 + (e & 1);
        float x = s[j][e] * scale_log2;
        if (key >= kvalid) x = -INFINITY;
        s[j][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_r[r], mx[r]);
      alpha[r] = exp2f(m_r[r] - m_new);
      m_r[r] = m_new;
      l_r[r] *= alpha[r];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[j][e] - m_r[e >> 1]);
        s[j][e] = p;
        l_r[e >> 1] += p;
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      acc[j][0] *= alpha[0];
      acc[j][1] *= alpha[0];
      acc[j][2] *= alpha[1];
      acc[j][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        uint32_t b[4];
        ldsm_x4_t(sv(st) + swz(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4)),
                  b);
        mma16816(acc[2 * dp], pa, b[0], b[1]);
        mma16816(acc[2 * dp + 1], pa, b[2], b[3]);
      }
    }
    __syncthreads();
  }

  // finish: reduce l over the quad, normalise, write
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int lr = warp * 16 + (lane >> 2) + r * 8;
    if (lr >= q_rows) continue;
    const long long grow = row0 + lr;
    const float inv = l_r[r] > 0.f ? 1.f / l_r[r] : 0.f;
    if (n_splits == 1) {
      __nv_bfloat16* od = o + grow * ld + h * D;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int col = j * 8 + (lane & 3) * 2;
        *reinterpret_cast<__nv_bfloat162*>(od + col) =
            __floats2bfloat162_rn(acc[j][2 * r] * inv, acc[j][2 * r + 1] * inv);
      }
    } else {
      float* od = o_part + ((long long)split * total_rows + grow) * ld + h * D;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int col = j * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2*>(od + col) =
            make_float2(acc[j][2 * r] * inv, acc[j][2 * r + 1] * inv);
      }
      if ((lane & 3) == 0)
        lse_part[((long long)split * total_rows + grow) * H + h] =
            l_r[r] > 0.f ? m_r[r] + log2f(l_r[r]) : -INFINITY;
    }
  }
}
}  // namespace fa

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
  for (int t = 0; t < a.nkeys[sess]; ++t) {
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
__global__ void attn_merge_kernel(const float* __restrict__ o_part,
                                  const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ o,
                                  long long total_rows, int H, int n_splits) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= total_rows * H) return;
  const long long row = gw / H;
  const int h = (int)(gw - row * H);
  float mmax = -INFINITY;
  for (int s = 0; s < n_splits; ++s)
    mmax = fmaxf(mmax, lse_part[((long long)s * total_rows + row) * H + h]);
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long ld = (long long)H * 128;
  for (int s = 0; s < n_splits; ++s) {
    const float lse = lse_part[((long long)s * total_rows + row) * H + h];
    if (lse == -INFINITY) continue;
    const float w = exp2f(lse - mmax);
    wsum += w;
    const float4 p = reinterpret_cast<const float4*>(o_part + ((long long)s * total_rows + row) * ld +
                                                     h * 128)[lane];
    acc.x = fmaf(w, p.x, acc.x);
    acc.y = fmaf(w, p.y, acc.y);
    acc.z = fmaf(w, p.z, acc.z);
    acc.w = fmaf(w, p.w, acc.w);
  }
  const float inv = 1.f / wsum;
  __nv_bfloat16* od = o + row * ld + h * 128 + lane * 4;
  *reinterpret_cast<__nv_bfloat162*>(od) = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  *reinterpret_cast<__nv_bfloat162*>(od + 2) = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
}

int attention_splits(int rows_per_session, int n_sessions, long long max_keys, int n_heads) {
  const int slots = 148 * 2;
  const long long ctas = (long long)n_sessions * ((rows_per_session + fa::BQ - 1) / fa::BQ) * n_heads;
  const long long tiles = (max_keys + fa::BKV - 1) / fa::BKV;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= kMaxSplits; ++s) {
    if (s > 1 && tiles / s < 4) break;
    const long long work = ctas * s;
    const long long waves = (work + slots - 1) / slots;
    const double eff = (double)work / (double)(waves * slots);
    // prefer fewer splits unless the wave fill improves by more than 5%
    if (eff > best_eff + 0.05) {
      best = s;
      best_eff = eff;
    }
  }
  return best;
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
  if (dtype == SFM_DTYPE_FP32) {
    ProfScope ps(SFM_PROF_ATTN, s);
    const long long warps = total_rows * n_heads;
    attn_f32_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(
        a, (const float*)q, (const float*)k, (const float*)v, (float*)o, n_heads, head_dim,
        scale_log2, total_rows);
    return record_cuda(cudaGetLastError());
  }
  if (head_dim != fa::D) return SFM_EUNSUPPORTED;
  const int qtiles = (a.rows_per + fa::BQ - 1) / fa::BQ;
  dim3 grid(a.n * qtiles, n_heads, n_splits);
  cudaFuncSetAttribute(fa::fa_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::SMEM);
  int rc;
  {
    ProfScope ps(SFM_PROF_ATTN, s);
    fa::fa_fwd_kernel<<<grid, fa::THREADS, fa::SMEM, s>>>(
        a, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (__nv_bfloat16*)o, o_part, lse_part, n_heads, n_splits, qtiles, scale_log2, total_rows);
    rc = record_cuda(cudaGetLastError());
  }
  if (rc || n_splits == 1) return rc;
  ProfScope ps(SFM_PROF_ATTN_MERGE, s);
  return launch_attention_merge(o_part, lse_part, o, total_rows, n_heads, n_splits, s);
}

int launch_attention_merge(const float* o_part, const float* lse_part, void* o,
                           long long total_rows, int n_heads, int n_splits, cudaStream_t s) {
  const long long warps = total_rows * n_heads;
  attn_merge_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(
      o_part, lse_part, (__nv_bfloat16*)o, total_rows, n_heads, n_splits);
  return record_cuda(cudaGetLastError());
}

}  // namespace sfm
