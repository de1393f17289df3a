// Row-wise and elementwise steps of f_theta and the Euler update.
//
//   embed        x_j = W_in z_j + e_mod[m(j)] + temb(tau)        (fp32 residual stream)
//   rmsnorm      x / sqrt(mean(x^2) + eps) * g -> GEMM operand dtype
//   rope_table   cos/sin of p * theta^(-2i/D_h), evaluated in fp64 once per call
//   rope_scatter rotate q, k (rotate-half pairs), q -> Q buffer, k/v -> the
//                session's cache rows after its valid cache (current unit's
//                scratch rows: the noisy unit is never committed to history,
//                "Wan-Streamer" v0.1 blog §3.4, clean context)
//   head_euler   v = RMSNorm(x; g_f) W_out^T ; z <- z + dtau * v   (§3.4 Euler)
//   euler        z <- z + dtau * v (vectorised, standalone)
#include "common.cuh"

namespace sfm {

struct PtrTable {
  float* p[kMaxBatch];
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// embed: one thread per column i, a strip of rows per CTA.  The tau embedding
// is evaluated in fp64 (angles reach 1000 rad).
// ---------------------------------------------------------------------------
constexpr int kEmbedRows = 32;

template <typename T>
__global__ void embed_kernel(BatchDesc b, PtrTable z, const T* __restrict__ w_in,
                             const T* __restrict__ e_mod, float tau, float* __restrict__ x, int d,
                             int c_lat) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d) return;
  const int half = d / 2;
  const int ii = i < half ? i : i - half;
  const double w = pow(10000.0, -2.0 * (double)ii / (double)d);
  const double ang = 1000.0 * (double)tau * w;
  const float te = (float)(i < half ? sin(ang) : cos(ang));
  float wr[64];
#pragma unroll 16
  for (int c = 0; c < c_lat; ++c) wr[c] = to_f(w_in[(size_t)i * c_lat + c]);
  const float em_v = to_f(e_mod[i]);
  const float em_a = to_f(e_mod[d + i]);
  const int rows = b.n * b.n_tok;
  const int r0 = blockIdx.y * kEmbedRows;
  for (int r = r0; r < r0 + kEmbedRows && r < rows; ++r) {
    const int sess = r / b.n_tok;
    const int j = r - sess * b.n_tok;
    const float* zr = z.p[sess] + (size_t)j * c_lat;
    float acc = 0.f;
#pragma unroll 16
    for (int c = 0; c < c_lat; ++c) acc = fmaf(zr[c], wr[c], acc);
    x[(size_t)r * d + i] = acc + (j < b.n_video ? em_v : em_a) + te;
  }
}

int launch_embed(const BatchDesc& b, float* const* z, const void* w_in, const void* e_mod,
                 float tau, float* x, int d, int c_lat, int dtype, cudaStream_t s) {
  PtrTable t{};
  for (int i = 0; i < b.n; ++i) t.p[i] = z[i];
  const int rows = b.n * b.n_tok;
  dim3 grid((d + 127) / 128, (rows + kEmbedRows - 1) / kEmbedRows);
  if (dtype == SFM_DTYPE_BF16)
    embed_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(b, t, (const __nv_bfloat16*)w_in,
                                                     (const __nv_bfloat16*)e_mod, tau, x, d, c_lat);
  else
    embed_kernel<float><<<grid, 128, 0, s>>>(b, t, (const float*)w_in, (const float*)e_mod, tau,
                                             x, d, c_lat);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// RMSNorm: one warp per row, float4 loads.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rmsnorm_kernel(const float* __restrict__ x, const T* __restrict__ g,
                               T* __restrict__ out, int rows, int d, float eps) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * d);
  const int nv = d / 4;
  float ss = 0.f;
  for (int c = lane; c < nv; c += 32) {
    const float4 a = xr[c];
    ss = fmaf(a.x, a.x, ss);
    ss = fmaf(a.y, a.y, ss);
    ss = fmaf(a.z, a.z, ss);
    ss = fmaf(a.w, a.w, ss);
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)d + eps);
  T* o = out + (size_t)row * d;
  for (int c = lane; c < nv; c += 32) {
    const float4 a = xr[c];
    o[4 * c + 0] = from_f<T>(a.x * r * to_f(g[4 * c + 0]));
    o[4 * c + 1] = from_f<T>(a.y * r * to_f(g[4 * c + 1]));
    o[4 * c + 2] = from_f<T>(a.z * r * to_f(g[4 * c + 2]));
    o[4 * c + 3] = from_f<T>(a.w * r * to_f(g[4 * c + 3]));
  }
}

int launch_rmsnorm(const float* x, const void* g, void* out, int rows, int d, float eps,
                   int dtype, cudaStream_t s) {
  const int blocks = (rows + 7) / 8;
  if (dtype == SFM_DTYPE_BF16)
    rmsnorm_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(x, (const __nv_bfloat16*)g,
                                                         (__nv_bfloat16*)out, rows, d, eps);
  else
    rmsnorm_kernel<float><<<blocks, 256, 0, s>>>(x, (const float*)g, (float*)out, rows, d, eps);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// RoPE table: cos/sin [rows][D_h/2] for positions p0[sess] + j, in fp64.
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(BatchDesc b, float* __restrict__ cos_t, float* __restrict__ sin_t,
                                  int half, double theta) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int rows = b.n * b.n_tok;
  if (idx >= rows * half) return;
  const int r = idx / half;
  const int i = idx - r * half;
  const int sess = r / b.n_tok;
  const int j = r - sess * b.n_tok;
  const double pos = (double)(b.p0[sess] + j);
  const double w = pow(theta, -2.0 * (double)i / (double)(2 * half));
  double sn, cs;
  sincos(pos * w, &sn, &cs);
  cos_t[idx] = (float)cs;
  sin_t[idx] = (float)sn;
}

int launch_rope_table(const BatchDesc& b, float* cos_t, float* sin_t, int head_dim, double theta,
                      cudaStream_t s) {
  const int half = head_dim / 2;
  const int total = b.n * b.n_tok * half;
  rope_table_kernel<<<(total + 255) / 256, 256, 0, s>>>(b, cos_t, sin_t, half, theta);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// RoPE + scatter: qkv fp32 [rows][3 H D] -> q [rows][H][D]; k, v -> cache rows
// base + valid + j of this layer.  One thread per (row, head, pair i).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rope_scatter_kernel(BatchDesc b, const float* __restrict__ qkv,
                                    const float* __restrict__ cos_t,
                                    const float* __restrict__ sin_t, T* __restrict__ q_out,
                                    T* __restrict__ k_layer, T* __restrict__ v_layer, int H,
                                    int D) {
  const int half = D / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int rows = b.n * b.n_tok;
  if (idx >= (long long)rows * H * half) return;
  const int i = (int)(idx % half);
  const int h = (int)((idx / half) % H);
  const int r = (int)(idx / ((long long)half * H));
  const int sess = r / b.n_tok;
  const int j = r - sess * b.n_tok;
  const float c = cos_t[(size_t)r * half + i];
  const float sn = sin_t[(size_t)r * half + i];
  const int hd = H * D;
  const float* src = qkv + (size_t)r * 3 * hd + h * D;
  const float qa = src[i], qb = src[i + half];
  const float ka = src[hd + i], kb = src[hd + i + half];
  const float va = src[2 * hd + i], vb = src[2 * hd + i + half];
  T* qd = q_out + (size_t)r * hd + h * D;
  qd[i] = from_f<T>(qa * c - qb * sn);
  qd[i + half] = from_f<T>(qb * c + qa * sn);
  const long long krow = b.base[sess] + b.valid[sess] + j;
  T* kd = k_layer + krow * hd + h * D;
  T* vd = v_layer + krow * hd + h * D;
  kd[i] = from_f<T>(ka * c - kb * sn);
  kd[i + half] = from_f<T>(kb * c + ka * sn);
  vd[i] = from_f<T>(va);
  vd[i + half] = from_f<T>(vb);
}

int launch_rope_scatter(const BatchDesc& b, const float* qkv, const float* cos_t,
                        const float* sin_t, void* q_out, void* k_layer, void* v_layer,
                        int n_heads, int head_dim, int dtype, cudaStream_t s) {
  const long long total = (long long)b.n * b.n_tok * n_heads * (head_dim / 2);
  const unsigned blocks = (unsigned)((total + 255) / 256);
  if (dtype == SFM_DTYPE_BF16)
    rope_scatter_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        b, qkv, cos_t, sin_t, (__nv_bfloat16*)q_out, (__nv_bfloat16*)k_layer,
        (__nv_bfloat16*)v_layer, n_heads, head_dim);
  else
    rope_scatter_kernel<float><<<blocks, 256, 0, s>>>(b, qkv, cos_t, sin_t, (float*)q_out,
                                                      (float*)k_layer, (float*)v_layer, n_heads,
                                                      head_dim);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Velocity head fused with the Euler update: one warp per token row.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void head_euler_kernel(BatchDesc b, const float* __restrict__ x,
                                  const T* __restrict__ g, const T* __restrict__ w_out,
                                  PtrTable z, PtrTable v_out, float dtau, int d, int c_lat,
                                  float eps) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = b.n * b.n_tok;
  if (row >= rows) return;
  const int sess = row / b.n_tok;
  const int j = row - sess * b.n_tok;
  const float* xr = x + (size_t)row * d;
  float ss = 0.f;
  for (int i = lane; i < d; i += 32) ss = fmaf(xr[i], xr[i], ss);
  ss = warp_sum(ss);
  const float rinv = rsqrtf(ss / (float)d + eps);
  for (int c0 = 0; c0 < c_lat; c0 += 16) {
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float xn = xr[i] * rinv * to_f(g[i]);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (c0 + c < c_lat) acc[c] = fmaf(xn, to_f(w_out[(size_t)(c0 + c) * d + i]), acc[c]);
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = warp_sum(acc[c]);
    float mine = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (lane == c) mine = acc[c];
    const int ch = c0 + lane;
    if (lane < 16 && ch < c_lat) {
      float* zr = z.p[sess] + (size_t)j * c_lat;
      zr[ch] = fmaf(dtau, mine, zr[ch]);
      if (v_out.p[sess]) v_out.p[sess][(size_t)j * c_lat + ch] = mine;
    }
  }
}

int launch_head_euler(const BatchDesc& b, const float* x, const void* g, const void* w_out,
                      float* const* z, float* const* v_out, float dtau, int d, int c_lat,
                      float eps, int dtype, cudaStream_t s) {
  PtrTable zt{}, vt{};
  for (int i = 0; i < b.n; ++i) {
    zt.p[i] = z[i];
    vt.p[i] = v_out ? v_out[i] : nullptr;
  }
  const int rows = b.n * b.n_tok;
  const int blocks = (rows + 7) / 8;
  if (dtype == SFM_DTYPE_BF16)
    head_euler_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        b, x, (const __nv_bfloat16*)g, (const __nv_bfloat16*)w_out, zt, vt, dtau, d, c_lat, eps);
  else
    head_euler_kernel<float><<<blocks, 256, 0, s>>>(b, x, (const float*)g, (const float*)w_out,
                                                    zt, vt, dtau, d, c_lat, eps);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// standalone Euler update, float4 vectorised grid-stride (HBM bound: 12 B/elt).
// ---------------------------------------------------------------------------
__global__ void euler_kernel(float* __restrict__ z, const float* __restrict__ v, float dtau,
                             long long n) {
  const long long n4 = n / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  float4* z4 = reinterpret_cast<float4*>(z);
  const float4* v4 = reinterpret_cast<const float4*>(v);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = z4[i];
    const float4 w = __ldcs(v4 + i);
    a.x = fmaf(dtau, w.x, a.x);
    a.y = fmaf(dtau, w.y, a.y);
    a.z = fmaf(dtau, w.z, a.z);
    a.w = fmaf(dtau, w.w, a.w);
    __stcs(z4 + i, a);
  }
  const long long t = n4 * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) z[t] = fmaf(dtau, v[t], z[t]);
}

int launch_euler(float* z, const float* v, float dtau, long long n, cudaStream_t s) {
  if (n <= 0) return SFM_OK;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long n4 = n / 4;
  long long blocks = (n4 + 511) / 512;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  euler_kernel<<<(unsigned)blocks, 512, 0, s>>>(z, v, dtau, n);
  return record_cuda(cudaGetLastError());
}

}  // namespace sfm
