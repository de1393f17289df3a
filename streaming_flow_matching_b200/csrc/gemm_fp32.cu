// Dense projections C = A B^T of f_theta (QKV, O, MLP-up, MLP-down) in the
// fp32 mode: CUDA-core SIMT kernel, 64x64x16 tiles (the fp32 mode's small
// shapes; bf16 projections run on the tensor cores in gemm_tc.cu).
//
// Epilogues: EPI_F32 store fp32; EPI_STORE store dtype; EPI_GELU store
// GELU_tanh(acc) as dtype; EPI_RESID C_fp32 += acc (residual stream).
#include "common.cuh"

namespace sfm {

__device__ __forceinline__ float gelu_tanh(float x) {
  const float k = 0.7978845608028654f;  // sqrt(2 / pi)
  return 0.5f * x * (1.f + tanhf(k * (x + 0.044715f * x * x * x)));
}

template <int EPI, typename T>
__device__ __forceinline__ void epi_pair(void* C, int ldc, int row, int col, float v0, float v1) {
  if (EPI == EPI_F32) {
    *reinterpret_cast<float2*>((float*)C + (size_t)row * ldc + col) = make_float2(v0, v1);
  } else if (EPI == EPI_RESID) {
    float2* p = reinterpret_cast<float2*>((float*)C + (size_t)row * ldc + col);
    float2 a = *p;
    a.x += v0;
    a.y += v1;
    *p = a;
  } else {
    if (EPI == EPI_GELU) {
      v0 = gelu_tanh(v0);
      v1 = gelu_tanh(v1);
    }
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<__nv_bfloat162*>((__nv_bfloat16*)C + (size_t)row * ldc + col) =
          __floats2bfloat162_rn(v0, v1);
    } else {
      *reinterpret_cast<float2*>((float*)C + (size_t)row * ldc + col) = make_float2(v0, v1);
    }
  }
}

// ---------------------------------------------------------------------------
// fp32 SIMT kernel
// ---------------------------------------------------------------------------
namespace simt {
constexpr int BM = 64, BN = 64, BK = 16;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A,
                                                       const float* __restrict__ B, void* C,
                                                       int M, int N, int K) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    // 64 rows x 16 k per operand = 1024 values, 4 per thread
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = tid + it * 256;
      const int r = e >> 4, kk = e & 15;
      const int ar = m0 + r;
      As[kk][r] = ar < M ? A[(size_t)ar * K + k0 + kk] : 0.f;
      Bs[kk][r] = B[(size_t)(n0 + r) * K + k0 + kk];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty * 4 + i;
    if (row >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j += 2)
      epi_pair<EPI, float>(C, N, row, n0 + tx * 4 + j, acc[i][j], acc[i][j + 1]);
  }
}
}  // namespace simt

int launch_gemm(const void* A, const void* B, void* C, int M, int N, int K, int epi, int dtype,
                cudaStream_t s) {
  if (M <= 0) return SFM_OK;
  if (dtype != SFM_DTYPE_FP32) return SFM_EUNSUPPORTED;   // bf16 runs on tcgen05 (gemm_tc.cu)
  {
    using namespace simt;
    if (N % BN || K % BK) return SFM_EUNSUPPORTED;
    dim3 grid(N / BN, (M + BM - 1) / BM);
    auto A32 = (const float*)A;
    auto B32 = (const float*)B;
    switch (epi) {
      case EPI_F32: gemm_f32_kernel<EPI_F32><<<grid, 256, 0, s>>>(A32, B32, C, M, N, K); break;
      case EPI_GELU: gemm_f32_kernel<EPI_GELU><<<grid, 256, 0, s>>>(A32, B32, C, M, N, K); break;
      case EPI_RESID: gemm_f32_kernel<EPI_RESID><<<grid, 256, 0, s>>>(A32, B32, C, M, N, K); break;
      case EPI_STORE: gemm_f32_kernel<EPI_STORE><<<grid, 256, 0, s>>>(A32, B32, C, M, N, K); break;
      default: return SFM_EINVAL;
    }
  }
  return record_cuda(cudaGetLastError());
}

}  // namespace sfm
