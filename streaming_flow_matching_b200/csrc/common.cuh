// Internal definitions shared by the kernels and the C-ABI of libsfm.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "sfm.h"

namespace sfm {

// Largest batch of sessions one call can carry (kernel parameters hold the
// per-session table by value, so batched launches stay graph-capturable).
constexpr int kMaxBatch = 16;

// Per-call description of the sessions in a batch; row r of the activations
// belongs to session r / n_tok, token r % n_tok.
struct BatchDesc {
  int n;                     // sessions in the batch
  int n_tok;                 // N: tokens of one unit
  int n_video;               // video tokens (the rest are audio)
  long long base[kMaxBatch]; // first pool row of each session's region
  int valid[kMaxBatch];      // S_c: valid cached tokens
  long long p0[kMaxBatch];   // position of the unit's first token
  int per_tau;               // 1: entry i is at flow time tau[i] (else one tau per call)
  float tau[kMaxBatch];
  long long t_unit[kMaxBatch]; // the unit's index on the timeline (3-D rotary embedding)
};

// Bounded-wait settings of the tensor-core kernels: the device word in which a
// timed-out wait records its site, the bound of every wait (1 s unless a test
// shortens it), and the test-only fault (SFM_FAULT_* bits) to inject.
struct Guard {
  int* err = nullptr;
  unsigned long long wait_ns = 1000000000ull;
  int fault = 0;
};

struct Session {
  bool open = false;
  int cache_units = 0;
  long long base_row = 0;
  long long units = 0;
};

int record_cuda(cudaError_t e);  // stores e for sfm_last_cuda_error; returns SFM_ECUDA or SFM_OK
// The calling thread's current CUDA context (CUcontext, NULL before the runtime has
// brought one up), through the driver entry point the runtime exposes.
int current_context(void** ctx);
void count_launch();             // one more kernel launched by this library

// Records a CUDA event pair around the launches in its scope when the
// profiler is on (sfm_profile_begin); no-op otherwise.
// True while sfm_profile_begin is in effect on this thread (launches are then
// issued directly, each bracketed by events, instead of through a CUDA graph).
bool profiling_active();

class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int idx_ = -1;
  cudaStream_t s_;
};

// Launch helpers (each returns 0 / SFM_ECUDA after checking cudaGetLastError).
// src_row_bytes / src_off_bytes: bytes per source row and offset of the copied
// part inside it (0, 0: the source rows are exactly the cache rows).
int launch_kv_append(const void* k, const void* v, void* k_pool, void* v_pool, int n_layers,
                     long long pool_tokens, int row_bytes, int n_tok, int unit_tokens,
                     long long base_row, long long first_unit, int cache_units, cudaStream_t s,
                     int src_row_bytes = 0, int src_off_bytes = 0);
int launch_kv_read(const void* k_pool, const void* v_pool, void* k_dst, void* v_dst, int layer,
                   long long pool_tokens, int row_bytes, long long row0, long long n_rows,
                   cudaStream_t s);

// With g (bf16 only): also xg = bf16(x g) and per-row partial sums of squares
// over 128-column blocks into ss ([rows][ss_ld]) -- the first RMSNorm, fused.
// Second half of a split-K residual projection (bf16 path): x += sum of the
// slices' partials ws[s][rows][d]; with g_next (bf16) also xg = bf16(x g) and
// the row's sum of squares into ss[row * ss_ld].
int launch_resid_splitk(float* x, const float* ws, int n_slices, int rows, int d,
                        const void* g_next, void* xg, float* ss, int ss_ld, cudaStream_t s);
int launch_embed(const BatchDesc& b, float* const* z, const void* w_in, const void* e_mod,
                 float tau, float* x, int d, int c_lat, int dtype, cudaStream_t s,
                 const void* g = nullptr, void* xg = nullptr, float* ss = nullptr, int ss_ld = 0);
int launch_rmsnorm(const float* x, const void* g, void* out, int rows, int d, float eps,
                   int dtype, cudaStream_t s);
// rope3d: (t, y, x) positions over a raster of grid_w columns (else p0 + j)
int launch_rope_table(const BatchDesc& b, float* cos_t, float* sin_t, int head_dim,
                      double theta, cudaStream_t s, bool rope3d = false, int grid_w = 1);
// SwiGLU on an fp32 [rows][2F] projection in the interleaved gate/up layout -> out [rows][F]
int launch_swiglu(const float* gu, void* out, int rows, int F, int dtype, cudaStream_t s);
int launch_rope_scatter(const BatchDesc& b, const float* qkv, const float* cos_t,
                        const float* sin_t, void* q_out, void* k_layer, void* v_layer,
                        int n_heads, int head_dim, int dtype, cudaStream_t s);
int launch_head_euler(const BatchDesc& b, const float* x, const void* g, const void* w_out,
                      float* const* z, float* const* v_out, float dtau, int d, int c_lat,
                      float eps, int dtype, cudaStream_t s, bool guided = false,
                      float scale = 1.f);
int launch_euler(float* z, const float* v, float dtau, long long n, cudaStream_t s);
int launch_exact_velocity_euler(float* z, const float* z0, float tau, float tau_next, long long n,
                                cudaStream_t s);

// GEMM C = A B^T, A [M][K], B [N][K] (both K-contiguous).
enum Epilogue { EPI_F32 = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_STORE = 3, EPI_QKV = 4, EPI_SWIGLU = 5 };
int launch_gemm(const void* A, const void* B, void* C, int M, int N, int K, int epi, int dtype,
                cudaStream_t s);

}  // namespace sfm
