// Dense projections C = A B^T of f_theta (QKV, O, MLP-up, MLP-down) on the
// CUDA cores / legacy MMA path.
//
//   bf16: mma.sync m16n8k16 (fp32 accumulate), 128x128x64 CTA tile, 3-stage
//         cp.async pipeline, XOR-swizzled shared memory.  This is the first,
//         correctness-first path; the tcgen05 path replaces it for the
//         large shapes.
//   fp32: CUDA-core SIMT 64x64x16 tile (the fp32 mode's small shapes).
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
// bf16 mma.sync kernel
// ---------------------------------------------------------------------------
namespace mma {
constexpr int BM = 128, BN = 128, BK = 64, STAGES = 3, THREADS = 256;
constexpr int TILE_BYTES = BM * BK * 2;  // 16 KB per operand tile
constexpr int SMEM = STAGES * 2 * TILE_BYTES;

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
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// byte offset of 16-byte chunk ch of row r in a [rows][64] bf16 tile (128 B rows)
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void load_tile(uint32_t sbase, const __nv_bfloat16* g, int rows_valid,
                                          int ld, int k0, int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int c = tid + it * THREADS;
    const int r = c >> 3, ch = c & 7;
    const bool ok = r < rows_valid;
    const __nv_bfloat16* src = g + (size_t)(ok ? r : 0) * ld + k0 + ch * 8;
    cp_async16(sbase + swz(r, ch), src, ok);
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS) gemm_bf16_kernel(const __nv_bfloat16* __restrict__ A,
                                                            const __nv_bfloat16* __restrict__ B,
                                                            void* C, int M, int N, int K) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const uint32_t sb = smem_u32(smem);
  const __nv_bfloat16* Ag = A + (size_t)m0 * K;
  const __nv_bfloat16* Bg = B + (size_t)n0 * K;
  const int a_rows = min(BM, M - m0);
  const int KT = K / BK;

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < KT) {
      load_tile(sb + s * 2 * TILE_BYTES, Ag, a_rows, K, s * BK, tid);
      load_tile(sb + s * 2 * TILE_BYTES + TILE_BYTES, Bg, BN, K, s * BK, tid);
    }
    cp_commit();
  }

  for (int kt = 0; kt < KT; ++kt) {
    cp_wait<STAGES - 2>();
    __syncthreads();
    const int pf = kt + STAGES - 1;
    if (pf < KT) {
      const int st = pf % STAGES;
      load_tile(sb + st * 2 * TILE_BYTES, Ag, a_rows, K, pf * BK, tid);
      load_tile(sb + st * 2 * TILE_BYTES + TILE_BYTES, Bg, BN, K, pf * BK, tid);
    }
    cp_commit();
    const uint32_t sa = sb + (kt % STAGES) * 2 * TILE_BYTES;
    const uint32_t sbb = sa + TILE_BYTES;
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      uint32_t af[4][4], bf[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = wm * 64 + i * 16 + (lane & 15);
        ldsm_x4(sa + swz(r, kk * 2 + (lane >> 4)), af[i][0], af[i][1], af[i][2], af[i][3]);
      }
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int r = wn * 32 + p * 16 + ((lane >> 4) << 3) + (lane & 7);
        ldsm_x4(sbb + swz(r, kk * 2 + ((lane >> 3) & 1)), bf[2 * p][0], bf[2 * p][1],
                bf[2 * p + 1][0], bf[2 * p + 1][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) mma16816(acc[i][j], af[i], bf[j]);
    }
  }
  cp_wait<0>();

#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = m0 + wm * 64 + i * 16 + (lane >> 2);
      const int col = n0 + wn * 32 + j * 8 + (lane & 3) * 2;
      if (row < M) epi_pair<EPI, __nv_bfloat16>(C, N, row, col, acc[i][j][0], acc[i][j][1]);
      if (row + 8 < M) epi_pair<EPI, __nv_bfloat16>(C, N, row + 8, col, acc[i][j][2], acc[i][j][3]);
    }
  }
}
}  // namespace mma

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
  if (dtype == SFM_DTYPE_BF16) {
    using namespace mma;
    if (N % BN || K % BK) return SFM_EUNSUPPORTED;
    dim3 grid(N / BN, (M + BM - 1) / BM);
    auto A16 = (const __nv_bfloat16*)A;
    auto B16 = (const __nv_bfloat16*)B;
    switch (epi) {
#define SFM_GEMM_CASE(E)                                                                \
  case E:                                                                               \
    cudaFuncSetAttribute(gemm_bf16_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                         SMEM);                                                         \
    gemm_bf16_kernel<E><<<grid, THREADS, SMEM, s>>>(A16, B16, C, M, N, K);              \
    break;
      SFM_GEMM_CASE(EPI_F32)
      SFM_GEMM_CASE(EPI_GELU)
      SFM_GEMM_CASE(EPI_RESID)
      SFM_GEMM_CASE(EPI_STORE)
#undef SFM_GEMM_CASE
      default:
        return SFM_EINVAL;
    }
  } else {
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
