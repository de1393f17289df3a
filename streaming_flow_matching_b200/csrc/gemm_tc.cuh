// tcgen05 GEMM launch interface.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace sfm {

struct GemmArgs {
  int M, N, K;
  int epi;               // Epilogue
  void* C;               // output (EPI_F32 / EPI_STORE / EPI_GELU) or fp32 residual (EPI_RESID)
  int ldc;
  int* err;              // device error word (bounded-wait timeouts)
  unsigned long long wait_ns;   // bound of every wait (0: 1 s)
  int fault;             // SFM_FAULT_GEMM_NO_LOADS: the producers issue no loads (test only)
  // EPI_QKV
  const float* cos_t;    // [M][64]
  const float* sin_t;
  __nv_bfloat16* q_out;  // [M][hd]
  __nv_bfloat16* k_layer;  // cache pool rows of this layer, [rows][hd]
  __nv_bfloat16* v_layer;
  int hd;
  BatchDesc b;
  int block_n;           // N-tile width the B tensor map was built for
  int pair;              // 1: CTA pairs (the B map's box has block_n / 2 rows)
  // RMSNorm of the updated residual, split across two GEMMs (bf16 path).
  // EPI_RESID with g_next: also writes xg = bf16(x * g_next) and, per row and
  // N tile, the partial sum of squares of the updated x: ss_out[row][n0 / BN].
  const __nv_bfloat16* g_next;
  __nv_bfloat16* xg;     // [M][N]
  float* ss_out;         // [M][ss_ld]
  // EPI_QKV / EPI_GELU with ss_in: A holds bf16(x * g); each accumulator row is
  // scaled by rsqrt(sum_{t < ss_n} ss_in[row][t] / norm_d + norm_eps).
  const float* ss_in;    // [M][ss_ld]
  int ss_n;
  int ss_ld;
  int norm_d;
  float norm_eps;
  // split-K (EPI_F32 only): unit u covers tile u % tiles and k-blocks of slice
  // u / tiles; slice s writes its fp32 partial to C + s * M * ldc
  int k_splits;          // 0 or 1: no split
};

// Whether an M x N projection runs on CTA pairs (256-row tiles, half of each B
// tile per CTA): M above 128 and at least 1.5 tiles per pair.
bool gemm_tc_pair(int M, int N, int hd, int epi, int sms);
// N-tile width (256, 192 or 128) for an M x N problem on `sms` SMs, in the given
// mode; 0 if none fits.
int gemm_tc_block_n(int M, int N, int hd, int epi, int sms, bool pair);
// K slices for a projection whose tiles fill under half of the SMs (single-CTA
// mode, at least 4 k-blocks per slice); 1 when no split pays.
int gemm_tc_k_splits(int M, int N, int K, int block_n, int sms);
// A: tensor map over [M_alloc][K] bf16, box {64, 128}; B: over [N][K], box
// {64, pair ? block_n / 2 : block_n}.
int launch_gemm_tc(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, int sms,
                   cudaStream_t s);

}  // namespace sfm
