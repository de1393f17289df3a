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

// CL: compile-time bound on c_lat (16, or 64 for any c_lat <= 64), so the
// W_in row stays in registers.  With g (bf16 path) the kernel also writes the
// first RMSNorm's numerator xg = bf16(x g) and, per row and 128-column block,
// the partial sum of squares ss[row][blockIdx.x] (the QKV GEMM applies 1 / rms).
template <typename T, int CL>
__global__ void __launch_bounds__(128) embed_kernel(
    const __grid_constant__ BatchDesc b, const __grid_constant__ PtrTable z,
    const T* __restrict__ w_in, const T* __restrict__ e_mod, float tau, float* __restrict__ x,
    int d, int c_lat, const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ xg,
    float* __restrict__ ss, int ss_ld) {
  __shared__ float red[kEmbedRows][4];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const bool on = i < d;
  const int rows = b.n * b.n_tok;
  const int r0 = blockIdx.y * kEmbedRows;
  if (!on && !g) return;
  const int ic = on ? i : 0;
  const int half = d / 2;
  const int ii = ic < half ? ic : ic - half;
  const double w = pow(10000.0, -2.0 * (double)ii / (double)d);
  auto temb = [&](float t) {
    const double ang = 1000.0 * (double)t * w;
    return (float)(ic < half ? sin(ang) : cos(ang));
  };
  // one flow time per call, or (several units of a pass) one per batch entry
  float te = b.per_tau ? 0.f : temb(tau);
  int te_sess = -1;
  float wr[CL];
#pragma unroll
  for (int c = 0; c < CL; ++c) wr[c] = c < c_lat ? to_f(w_in[(size_t)ic * c_lat + c]) : 0.f;
  const float em_v = to_f(e_mod[ic]);
  const float em_a = to_f(e_mod[d + ic]);
  const float gi = g && on ? __bfloat162float(g[i]) : 0.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = 0; rr < kEmbedRows; ++rr) {
    const int r = r0 + rr;
    if (r >= rows) break;
    const int sess = r / b.n_tok;
    const int j = r - sess * b.n_tok;
    if (b.per_tau && sess != te_sess) {
      te = temb(b.tau[sess]);
      te_sess = sess;
    }
    const float* zr = z.p[sess] + (size_t)j * c_lat;
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < CL; ++c)
      if (c < c_lat) acc = fmaf(zr[c], wr[c], acc);
    const float xv = acc + (j < b.n_video ? em_v : em_a) + te;
    if (on) x[(size_t)r * d + i] = xv;
    if (g) {
      if (on) xg[(size_t)r * d + i] = __float2bfloat16_rn(xv * gi);
      const float sq = warp_sum(on ? xv * xv : 0.f);
      if (lane == 0) red[rr][warp] = sq;
    }
  }
  if (g) {
    __syncthreads();
    if (threadIdx.x < kEmbedRows && r0 + (int)threadIdx.x < rows) {
      const float* t = red[threadIdx.x];
      ss[(size_t)(r0 + threadIdx.x) * ss_ld + blockIdx.x] = (t[0] + t[1]) + (t[2] + t[3]);
    }
  }
}

int launch_embed(const BatchDesc& b, float* const* z, const void* w_in, const void* e_mod,
                 float tau, float* x, int d, int c_lat, int dtype, cudaStream_t s,
                 const void* g, void* xg, float* ss, int ss_ld) {
  PtrTable t{};
  for (int i = 0; i < b.n; ++i) t.p[i] = z[i];
  const int rows = b.n * b.n_tok;
  dim3 grid((d + 127) / 128, (rows + kEmbedRows - 1) / kEmbedRows);
  if (c_lat > 64) return SFM_EUNSUPPORTED;
  const bool c16 = c_lat == 16;
  if (dtype == SFM_DTYPE_BF16) {
    auto k = c16 ? embed_kernel<__nv_bfloat16, 16> : embed_kernel<__nv_bfloat16, 64>;
    k<<<grid, 128, 0, s>>>(b, t, (const __nv_bfloat16*)w_in, (const __nv_bfloat16*)e_mod, tau, x,
                           d, c_lat, (const __nv_bfloat16*)g, (__nv_bfloat16*)xg, ss, ss_ld);
  } else {
    if (g) return SFM_EINVAL;    // the fused norm is a bf16-path feature
    auto k = c16 ? embed_kernel<float, 16> : embed_kernel<float, 64>;
    k<<<grid, 128, 0, s>>>(b, t, (const float*)w_in, (const float*)e_mod, tau, x, d, c_lat, nullptr,
                           nullptr, nullptr, 0);
  }
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// RMSNorm: one CTA per row; each thread holds 8 consecutive elements in
// registers (one read of x), block reduction of the sum of squares, 16-byte
// stores of the bf16 (or 2 x 16-byte fp32) output.  d / 8 <= 1024.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void store8(__nv_bfloat16* o, const float* v) {
  uint4 u;
  __nv_bfloat162 t;
  t = __floats2bfloat162_rn(v[0], v[1]); u.x = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[2], v[3]); u.y = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[4], v[5]); u.z = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[6], v[7]); u.w = *reinterpret_cast<uint32_t*>(&t);
  *reinterpret_cast<uint4*>(o) = u;
}
__device__ __forceinline__ void store8(float* o, const float* v) {
  reinterpret_cast<float4*>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* v) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(1024) rmsnorm_kernel(const float* __restrict__ x,
                                                      const T* __restrict__ g,
                                                      T* __restrict__ out, int d, float eps) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  const int c = threadIdx.x * 8;
  const bool on = c < d;
  float v[8];
  float ss = 0.f;
  if (on) {
    load8(x + (size_t)row * d + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
  }
  ss = warp_sum(ss);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (warp == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[0] = t;
  }
  __syncthreads();
  if (!on) return;
  const float r = rsqrtf(red[0] / (float)d + eps);
  float gv[8];
  load8(g + c, gv);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = v[i] * r * gv[i];
  store8(out + (size_t)row * d + c, v);
}

// Split-K residual projection, second half: x += the K slices' partial
// products (ws[s][row][:], summed in slice order), and with g_next the next
// RMSNorm's numerator bf16(x g) and the row's sum of squares ss[row][0].
// One CTA per row, 8 columns per thread.
__global__ void __launch_bounds__(1024) resid_splitk_kernel(
    float* __restrict__ x, const float* __restrict__ ws, int n_slices, int rows, int d,
    const __nv_bfloat16* __restrict__ g_next, __nv_bfloat16* __restrict__ xg,
    float* __restrict__ ss, int ss_ld) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  const int c = threadIdx.x * 8;
  const bool on = c < d;
  float v[8];
  float sq = 0.f;
  if (on) {
    load8(x + (size_t)row * d + c, v);
    for (int sl = 0; sl < n_slices; ++sl) {
      float p[8];
      load8(ws + ((size_t)sl * rows + row) * d + c, p);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += p[i];
    }
    store8(x + (size_t)row * d + c, v);
    if (g_next) {
      float gv[8];
      load8(g_next + c, gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sq = fmaf(v[i], v[i], sq);
        v[i] *= gv[i];
      }
      store8(xg + (size_t)row * d + c, v);
    }
  }
  if (!g_next) return;
  sq = warp_sum(sq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = sq;
  __syncthreads();
  if (warp == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) ss[(size_t)row * ss_ld] = t;
  }
}

int launch_resid_splitk(float* x, const float* ws, int n_slices, int rows, int d,
                        const void* g_next, void* xg, float* ss, int ss_ld, cudaStream_t s) {
  if (rows <= 0) return SFM_OK;
  if (d % 8 || d / 8 > 1024) return SFM_EUNSUPPORTED;
  const int threads = ((d / 8) + 31) / 32 * 32;
  resid_splitk_kernel<<<rows, threads, 0, s>>>(x, ws, n_slices, rows, d,
                                              (const __nv_bfloat16*)g_next, (__nv_bfloat16*)xg,
                                              ss, ss_ld);
  return record_cuda(cudaGetLastError());
}

int launch_rmsnorm(const float* x, const void* g, void* out, int rows, int d, float eps,
                   int dtype, cudaStream_t s) {
  if (rows <= 0) return SFM_OK;
  if (d % 8 || d / 8 > 1024) return SFM_EUNSUPPORTED;
  const int threads = ((d / 8) + 31) / 32 * 32;
  if (dtype == SFM_DTYPE_BF16)
    rmsnorm_kernel<__nv_bfloat16><<<rows, threads, 0, s>>>(x, (const __nv_bfloat16*)g,
                                                          (__nv_bfloat16*)out, d, eps);
  else
    rmsnorm_kernel<float><<<rows, threads, 0, s>>>(x, (const float*)g, (float*)out, d, eps);
  return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// RoPE table: cos/sin [rows][D_h/2] for positions p0[sess] + j, in fp64.
// ---------------------------------------------------------------------------
// 3-D form (rope3d): pair i belongs to the time band (the first half - 2 ns pairs), the
// row band or the column band (ns = head_dim / 6 pairs each); within a band of n_b pairs,
// pair k turns by pos_axis * theta^(-k / n_b); positions (t_unit, y, x) for video token j
// = y grid_w + x, (t_unit, 0, 0) for audio.
__global__ void rope_table_kernel(BatchDesc b, float* __restrict__ cos_t, float* __restrict__ sin_t,
                                  int half, double theta, int rope3d, int grid_w) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int rows = b.n * b.n_tok;
  if (idx >= rows * half) return;
  const int r = idx / half;
  const int i = idx - r * half;
  const int sess = r / b.n_tok;
  const int j = r - sess * b.n_tok;
  double ang;
  if (rope3d) {
    const int ns = (2 * half) / 6, nt = half - 2 * ns;
    const bool video = j < b.n_video;
    double pos;
    int k, nb;
    if (i < nt) {
      pos = (double)b.t_unit[sess];
      k = i;
      nb = nt;
    } else if (i < nt + ns) {
      pos = video ? (double)(j / grid_w) : 0.0;
      k = i - nt;
      nb = ns;
    } else {
      pos = video ? (double)(j % grid_w) : 0.0;
      k = i - nt - ns;
      nb = ns;
    }
    ang = pos * pow(theta, -(double)k / (double)nb);
  } else {
    const double pos = (double)(b.p0[sess] + j);
    ang = pos * pow(theta, -2.0 * (double)i / (double)(2 * half));
  }
  double sn, cs;
  sincos(ang, &sn, &cs);
  cos_t[idx] = (float)cs;
  sin_t[idx] = (float)sn;
}

int launch_rope_table(const BatchDesc& b, float* cos_t, float* sin_t, int head_dim, double theta,
                      cudaStream_t s, bool rope3d, int grid_w) {
  const int half = head_dim / 2;
  const int total = b.n * b.n_tok * half;
  if (rope3d && grid_w < 1) return SFM_EINVAL;
  rope_table_kernel<<<(total + 255) / 256, 256, 0, s>>>(b, cos_t, sin_t, half, theta,
                                                        rope3d ? 1 : 0, grid_w);
  return record_cuda(cudaGetLastError());
}

// SwiGLU of an fp32 projection in the interleaved layout: column 128 b + c (c < 64) is gate
// unit 64 b + c and column 128 b + 64 + c its up partner; out = silu(gate) * up.
template <typename T>
__global__ void swiglu_kernel(const float* __restrict__ gu, T* __restrict__ out, long long n, int F) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const long long r = idx / F;
  const int f = (int)(idx - r * F);
  const float* row = gu + r * 2 * (long long)F;
  const int col = (f / 64) * 128 + (f % 64);
  const float g = row[col], u = row[col + 64];
  out[idx] = from_f<T>(g / (1.f + expf(-g)) * u);
}

int launch_swiglu(const float* gu, void* out, int rows, int F, int dtype, cudaStream_t s) {
  const long long n = (long long)rows * F;
  if (n == 0) return SFM_OK;
  if (F % 64) return SFM_EUNSUPPORTED;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dtype == SFM_DTYPE_BF16)
    swiglu_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(gu, (__nv_bfloat16*)out, n, F);
  else
    swiglu_kernel<float><<<blocks, 256, 0, s>>>(gu, (float*)out, n, F);
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
// Velocity head fused with the final RMSNorm and the Euler update.  One CTA of
// kHeadThreads per kHeadRows token rows: every thread walks a strided set of
// 4-column groups, accumulating sum(x^2) per row and x*g*W_out for 16 output
// channels per row, so the RMS scale is applied once to the finished dot
// products.  The 64 partial sums per thread are reduced across the warp by
// halving exchanges (each step hands half of the values to the partner lane),
// which leaves 2 totals per lane after 62 shuffles; warps then combine
// through shared memory.
//
// Guided (classifier-free guidance, "Wan-Streamer" v0.1 blog, training Stage 3):
// batch entries 2p and 2p + 1 are the conditional and unconditional evaluations
// at the same z.  A CTA then takes tokens j, j + 1 of both entries (its 4 rows),
// forms v = v_u + s (v_c - v_u) per token and updates entry 2p's z once.
// ---------------------------------------------------------------------------
constexpr int kHeadRows = 4, kHeadThreads = 256, kHeadCh = 16;
constexpr int kHeadVals = kHeadRows * kHeadCh;   // 64 accumulators per thread

__device__ __forceinline__ void load4(const float* p, float* o) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* o) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
}

template <int N>
__device__ __forceinline__ void halve_step(float* acc, int lane, int o) {
  const bool up = (lane & o) != 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float send = up ? acc[j] : acc[j + N];
    const float keep = up ? acc[j + N] : acc[j];
    acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

template <typename T, bool GUIDED>
__global__ void __launch_bounds__(kHeadThreads)
    head_euler_kernel(const __grid_constant__ BatchDesc b, const float* __restrict__ x, const T* __restrict__ g,
                      const T* __restrict__ w_out, const __grid_constant__ PtrTable z,
                      const __grid_constant__ PtrTable v_out, float dtau, int d,
                      int c_lat, float eps, float scale) {
  __shared__ float red[kHeadThreads / 32][kHeadVals];
  __shared__ float red_ss[kHeadThreads / 32][kHeadRows];
  __shared__ float vsh[GUIDED ? kHeadVals : 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the CTA's rows of x: consecutive rows, or (guided) tokens j0, j0 + 1 of the
  // conditional entry 2p followed by the same tokens of the unconditional entry
  long long xrow[kHeadRows];
  bool live[kHeadRows];
  int pair = 0, j0 = 0;
  if (GUIDED) {
    const int per_pair = (b.n_tok + 1) / 2;
    pair = blockIdx.x / per_pair;
    j0 = (blockIdx.x - pair * per_pair) * 2;
#pragma unroll
    for (int q = 0; q < kHeadRows; ++q) {
      const int j = j0 + (q & 1);
      live[q] = j < b.n_tok;
      xrow[q] = (long long)(2 * pair + (q >> 1)) * b.n_tok + (live[q] ? j : 0);
    }
  } else {
    const int rows = b.n * b.n_tok;
    const int row0 = blockIdx.x * kHeadRows;
#pragma unroll
    for (int q = 0; q < kHeadRows; ++q) {
      live[q] = row0 + q < rows;
      xrow[q] = live[q] ? row0 + q : row0;
    }
  }
  for (int c0 = 0; c0 < c_lat; c0 += kHeadCh) {
    const int nc = c_lat - c0 < kHeadCh ? c_lat - c0 : kHeadCh;
    float acc[kHeadVals];
    float ss[kHeadRows];
#pragma unroll
    for (int k = 0; k < kHeadVals; ++k) acc[k] = 0.f;
#pragma unroll
    for (int q = 0; q < kHeadRows; ++q) ss[q] = 0.f;
    for (int i = 4 * threadIdx.x; i < d; i += 4 * kHeadThreads) {
      float gi[4], xv[kHeadRows][4];
      load4(g + i, gi);
#pragma unroll
      for (int q = 0; q < kHeadRows; ++q) {
        if (live[q]) {
          load4(x + (size_t)xrow[q] * d + i, xv[q]);
        } else {
          xv[q][0] = xv[q][1] = xv[q][2] = xv[q][3] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ss[q] = fmaf(xv[q][e], xv[q][e], ss[q]);
          xv[q][e] *= gi[e];
        }
      }
#pragma unroll
      for (int c = 0; c < kHeadCh; ++c) {
        float wv[4] = {0.f, 0.f, 0.f, 0.f};
        if (c < nc) load4(w_out + (size_t)(c0 + c) * d + i, wv);
#pragma unroll
        for (int q = 0; q < kHeadRows; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q * kHeadCh + c] = fmaf(xv[q][e], wv[e], acc[q * kHeadCh + c]);
      }
    }
    // halving exchange: after the step with offset o a lane keeps the half of
    // its values selected by (lane & o); lane L ends holding totals 2L, 2L+1
    halve_step<32>(acc, lane, 16);
    halve_step<16>(acc, lane, 8);
    halve_step<8>(acc, lane, 4);
    halve_step<4>(acc, lane, 2);
    halve_step<2>(acc, lane, 1);
#pragma unroll
    for (int q = 0; q < kHeadRows; ++q) ss[q] = warp_sum(ss[q]);
    red[warp][2 * lane] = acc[0];
    red[warp][2 * lane + 1] = acc[1];
    if (lane < kHeadRows) {
      float mine = ss[0];
#pragma unroll
      for (int q = 1; q < kHeadRows; ++q)
        if (lane == q) mine = ss[q];
      red_ss[warp][lane] = mine;
    }
    __syncthreads();
    if (threadIdx.x < kHeadVals) {
      const int q = threadIdx.x / kHeadCh, c = threadIdx.x % kHeadCh;
      float dot = 0.f, sq = 0.f;
#pragma unroll
      for (int w = 0; w < kHeadThreads / 32; ++w) {
        dot += red[w][threadIdx.x];
        sq += red_ss[w][q];
      }
      const float v = dot * rsqrtf(sq / (float)d + eps);
      if (GUIDED) {
        vsh[threadIdx.x] = v;
      } else if (blockIdx.x * kHeadRows + q < b.n * b.n_tok && c < nc) {
        const int row = blockIdx.x * kHeadRows + q;
        const int sess = row / b.n_tok;
        const int j = row - sess * b.n_tok;
        float* zr = z.p[sess] + (size_t)j * c_lat + c0 + c;
        if (dtau != 0.f) *zr = fmaf(dtau, v, *zr);   // a zero-length step only reports v
        if (v_out.p[sess]) v_out.p[sess][(size_t)j * c_lat + c0 + c] = v;
      }
    }
    if (GUIDED) {
      __syncthreads();
      // threads 0..31: token j0 + (t / 16), channel c0 + (t % 16)
      const int t = threadIdx.x, q = t / kHeadCh, c = t % kHeadCh;
      if (t < 2 * kHeadCh && j0 + q < b.n_tok && c < nc) {
        const float vc = vsh[q * kHeadCh + c], vu = vsh[(q + 2) * kHeadCh + c];
        const float v = fmaf(scale, vc - vu, vu);
        const int sess = 2 * pair, j = j0 + q;
        float* zr = z.p[sess] + (size_t)j * c_lat + c0 + c;
        *zr = fmaf(dtau, v, *zr);
        if (v_out.p[sess]) v_out.p[sess][(size_t)j * c_lat + c0 + c] = v;
      }
    }
    __syncthreads();
  }
}

int launch_head_euler(const BatchDesc& b, const float* x, const void* g, const void* w_out,
                      float* const* z, float* const* v_out, float dtau, int d, int c_lat,
                      float eps, int dtype, cudaStream_t s, bool guided, float scale) {
  PtrTable zt{}, vt{};
  for (int i = 0; i < b.n; ++i) {
    zt.p[i] = z[i];
    vt.p[i] = v_out ? v_out[i] : nullptr;
  }
  if (guided && (b.n % 2 || b.n_tok < 1)) return SFM_EINVAL;
  const int rows = b.n * b.n_tok;
  const int blocks = guided ? (b.n / 2) * ((b.n_tok + 1) / 2) : (rows + kHeadRows - 1) / kHeadRows;
  if (blocks == 0) return SFM_OK;
  if (d % 4 || ((uintptr_t)g & 15u) || ((uintptr_t)w_out & 15u) || ((uintptr_t)x & 15u))
    return SFM_EUNSUPPORTED;
  if (dtype == SFM_DTYPE_BF16) {
    auto k = guided ? head_euler_kernel<__nv_bfloat16, true> : head_euler_kernel<__nv_bfloat16, false>;
    k<<<blocks, kHeadThreads, 0, s>>>(b, x, (const __nv_bfloat16*)g, (const __nv_bfloat16*)w_out, zt,
                                      vt, dtau, d, c_lat, eps, scale);
  } else {
    auto k = guided ? head_euler_kernel<float, true> : head_euler_kernel<float, false>;
    k<<<blocks, kHeadThreads, 0, s>>>(b, x, (const float*)g, (const float*)w_out, zt, vt, dtau, d,
                                      c_lat, eps, scale);
  }
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

// ---------------------------------------------------------------------------
// exact-velocity Euler step (closed-form check of the solve loop): on the
// rectified-flow path z_tau = (1 - tau) z0 + tau eps the velocity is
// eps - z0 = (z_tau - z0) / tau, so a step evaluated at tau_i with that state-
// dependent velocity stays on the path, and the solve ends at z0 for any schedule.
// ---------------------------------------------------------------------------
__global__ void exact_velocity_euler_kernel(float* __restrict__ z, const float* __restrict__ z0,
                                            float inv_tau, float dtau, long long n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float zi = z[i];
    const float v = (zi - z0[i]) * inv_tau;
    z[i] = fmaf(dtau, v, zi);
  }
}

int launch_exact_velocity_euler(float* z, const float* z0, float tau, float tau_next, long long n,
                                cudaStream_t s) {
  if (n <= 0) return SFM_OK;
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  exact_velocity_euler_kernel<<<(unsigned)blocks, 256, 0, s>>>(z, z0, 1.f / tau, tau_next - tau, n);
  return record_cuda(cudaGetLastError());
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
