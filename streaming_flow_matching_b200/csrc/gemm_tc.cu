// Dense projections of f_theta on the 5th-generation tensor cores (tcgen05):
//   C[M][N] = A[M][K] . B[N][K]^T,  A = activations (bf16), B = weights (bf16,
//   stored [out][in]), fp32 accumulation in tensor memory.
//
// Persistent, warp-specialised CTA (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 per stage
//               (128-byte swizzle), STAGES-deep ring of shared-memory stages
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//               into one of two TMEM accumulators and commits to mbarriers
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (thread = row), fused
//               epilogue, global stores; the other accumulator is being filled
//               meanwhile
// Pair mode (two CTAs of a cluster on neighbouring SMs, tcgen05 cta_group::2):
// a 256-row tile, rows [0,128) in the even CTA and [128,256) in the odd one; each
// CTA stages its own A rows and half of the B tile (BN/2 weight rows), so every
// weight byte reaches shared memory once per pair instead of once per CTA.  Both
// CTAs' loads of a stage complete on the even CTA's barrier (which expects the
// bytes of both); the even CTA's lane issues the M = 256 MMAs and its commits
// arrive on both CTAs' barriers; each CTA's epilogue drains its own 128
// accumulator rows.
// Epilogues: EPI_F32 / EPI_STORE / EPI_GELU / EPI_RESID (x += acc, fp32) and
// EPI_QKV: rotary embedding of q and k in fp32 (rotate-half pairs (i, i+64) of
// each 128-wide head), q to the Q buffer, k and v to the sessions' cache rows
// after their valid cache (the current unit's scratch rows).
#include "gemm_tc.cuh"
#include "sm100.cuh"

namespace sfm {

using namespace sm100;

namespace gtc {

constexpr int BM = 128, BK = 64;
constexpr int THREADS = 192;

template <int BN, bool PAIR> struct Cfg {
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;   // weight rows staged by this CTA
  static constexpr int STAGES = PAIR ? (BN == 256 ? 6 : (BN == 192 ? 7 : 8))
                                     : (BN == 256 ? 4 : (BN == 192 ? 5 : 6));
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = BN == 128 ? 128 : 256;     // TMEM columns between the two accumulators
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  // after the stages: 256 B of barriers, then the epilogue's transpose buffers
  // (4 warps x 32 rows x 32 fp32), then alignment slack
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES + 256;
  static constexpr int EPI_BYTES = 4 * 32 * 32 * 4;
  static constexpr int SMEM = EPI_OFF + EPI_BYTES + 1024;
};

__device__ __forceinline__ float gelu_tanh(float x) {
  const float k = 0.7978845608028654f;
  return 0.5f * x * (1.f + tanhf(k * (x + 0.044715f * x * x * x)));
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}

template <int BN, int EPI, bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b, const __grid_constant__ GemmArgs args) {
  using C = Cfg<BN, PAIR>;
  static_assert(C::STAGES <= 8, "producer bookkeeping holds 8 stages");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tiles of TM rows: 128 (one CTA) or 256 (a pair); unit = this CTA or pair
  constexpr int TM = PAIR ? 2 * BM : BM;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int m_tiles = (args.M + TM - 1) / TM;
  const int n_tiles = args.N / BN;
  const int tiles = m_tiles * n_tiles;
  const int kblocks = args.K / BK;
  const int ksp = args.k_splits > 1 ? args.k_splits : 1;
  const int units_total = tiles * ksp;       // (tile, k slice) work units
  const unsigned long long wait_ns = args.wait_ns ? args.wait_ns : kWaitNs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIR ? 8 : 4);   // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&map_a);
    tma_prefetch(&map_b);
  }
  tc_fence_before();
  if (PAIR) {
    __syncwarp();
    cluster_sync();        // both CTAs' barriers exist before any remote arrive
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && !(args.fault & SFM_FAULT_GEMM_NO_LOADS)) {
      // ---------------- TMA producer (its own A rows and B rows) ----------------
      int s = 0;
      uint32_t ph = 0;
      int last_parity[8];
      for (int i = 0; i < C::STAGES; ++i) last_parity[i] = -1;
      bool ok = true;
      for (int u = unit; u < units_total && ok; u += n_units) {
        const int t = u % tiles, sl = u / tiles;
        const int m0 = (t % m_tiles) * TM + (int)rank * BM;
        const int n0 = (t / m_tiles) * BN + (int)rank * C::B_ROWS;
        for (int kb = sl * kblocks / ksp; kb < (sl + 1) * kblocks / ksp; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort, args.err, 0x101, wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t sa = base + s * C::STAGE_BYTES;
          if (PAIR) {
            // both halves complete on the even CTA's barrier, which expects both
            const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sa, &map_a, bar, kb * BK, m0);
            tma_load_2d_pair(sa + C::A_BYTES, &map_b, bar, kb * BK, n0);
          } else {
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
            tma_load_2d(sa, &map_a, &full[s], kb * BK, m0);
            tma_load_2d(sa + C::A_BYTES, &map_b, &full[s], kb * BK, n0);
          }
          last_parity[s] = (int)ph;
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {  // unwinding: let the loads already issued land before the CTA exits
        if (PAIR && !leader) {
          // this CTA's loads complete on the even CTA's barrier: give them a bound
          const unsigned long long t0 = globaltimer();
          while (globaltimer() - t0 < 100000ull) {
          }
        } else {
          for (int i = 0; i < C::STAGES; ++i)
            if (last_parity[i] >= 0) mbar_drain(&full[i], (uint32_t)last_parity[i], wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the CTA, or the pair's even CTA) ----------------
      constexpr uint32_t idesc = idesc_bf16(TM, BN, false, false);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true, issued = false;
      for (int u = unit; u < units_total && ok; u += n_units) {
        const int sl = u / tiles;
        const int kb0 = sl * kblocks / ksp, kb1 = (sl + 1) * kblocks / ksp;
        if (!(PAIR ? mbar_wait_cluster(&acc_empty[acc], acc_ph ^ 1u, abort, args.err, 0x102, wait_ns)
                   : mbar_wait(&acc_empty[acc], acc_ph ^ 1u, abort, args.err, 0x102, wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * C::ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, abort, args.err, 0x103, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * C::STAGE_BYTES;
          const uint64_t da = sw128_desc(sa, 16, 1024);
          const uint64_t db = sw128_desc(sa + C::A_BYTES, 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {  // +32 bytes per K=16 step inside the swizzle atom
            if (PAIR)
              umma_bf16_pair(d, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc,
                             (kb != kb0 || k != 0) ? 1u : 0u);
            else
              umma_bf16(d, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc,
                        (kb != kb0 || k != 0) ? 1u : 0u);
          }
          issued = true;
          if (PAIR)
            umma_commit_pair(&empty[s], 3);
          else
            umma_commit(&empty[s]);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR)
          umma_commit_pair(&acc_full[acc], 3);
        else
          umma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1u;
      }
      if (!ok && issued) {  // unwinding: wait for the MMAs already issued
        if (PAIR)
          umma_commit_pair(drain, 1);
        else
          umma_commit(drain);
        mbar_drain(drain, 0, wait_ns);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5, thread = accumulator row) ----------------
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int u = unit; u < units_total; u += n_units) {
      const int t = u % tiles, sl = u / tiles;
      const int m0 = (t % m_tiles) * TM + (int)rank * BM, n0 = (t / m_tiles) * BN;
      const int row = m0 + quarter * 32 + lane;
      const bool live = row < args.M;
      // residual add, coalesced: the warp's 32 x 32 accumulator chunk goes through a
      // shared-memory transpose, and lane (cg = lane & 7, rsub = lane >> 3) then handles
      // float4 column group cg of rows 4 it + rsub (it = 0..7), so 8 lanes cover one
      // row's 128 contiguous bytes.  The residual of chunk 0 is loaded (from L2) while
      // the tile's MMAs finish; chunk c + 1 while chunk c is stored.
      const int cg = lane & 7, rsub = lane >> 3;
      const int wrow0 = m0 + quarter * 32;
      float4 res[2][8];
      auto load_res = [&](int c, float4* dst) {
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = wrow0 + 4 * it + rsub;
          if (rr < args.M)
            dst[it] = *reinterpret_cast<const float4*>((const float*)args.C + (size_t)rr * args.ldc + n0 +
                                                       c * 32 + cg * 4);
        }
      };
      if (EPI == EPI_RESID) {
        // the epilogue warps idle through the mainloop: pull this row's residual slice
        // into L2 now (it was written several kernels ago and may have left L2)
        if (live) prefetch_l2_bulk((const float*)args.C + (size_t)row * args.ldc + n0, BN * 4);
        load_res(0, res[0]);
      }
      // fused RMSNorm of the A rows: 1 / rms of this row from the producer's partial sums
      float rinv = 1.f;
      if ((EPI == EPI_QKV || EPI == EPI_GELU || EPI == EPI_SWIGLU) && args.ss_in && live) {
        float ss = 0.f;
        for (int t2 = 0; t2 < args.ss_n; ++t2) ss += args.ss_in[(size_t)row * args.ss_ld + t2];
        rinv = rsqrtf(ss / (float)args.norm_d + args.norm_eps);
      }
      if (!__all_sync(0xffffffffu, PAIR ? mbar_wait_cluster(&acc_full[acc], acc_ph, abort, args.err, 0x104, wait_ns)
                                        : mbar_wait(&acc_full[acc], acc_ph, abort, args.err, 0x104, wait_ns)))
        break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      if (EPI == EPI_QKV) {
        const int hd = args.hd;
        const int section = n0 / hd;           // 0 q, 1 k, 2 v (a tile never straddles)
        for (int hh = 0; hh < BN / 128; ++hh) {
          const int head = (n0 - section * hd) / 128 + hh;
          for (int half = 0; half < 2; ++half) {
            uint32_t ra[32], rb[32];
            tmem_ld32(tbase + hh * 128 + half * 32, ra);
            tmem_ld32(tbase + hh * 128 + 64 + half * 32, rb);
            tmem_wait_ld(ra);
            reg_fence(rb);
            if (row >= args.M) continue;
            float a[32], b[32];
            if (section < 2) {
              // this row's cos / sin for pairs [32 half, 32 half + 32): 16-byte loads
              const float4* cs = reinterpret_cast<const float4*>(args.cos_t + (size_t)row * 64 + half * 32);
              const float4* sn = reinterpret_cast<const float4*>(args.sin_t + (size_t)row * 64 + half * 32);
#pragma unroll
              for (int i4 = 0; i4 < 8; ++i4) {
                const float4 c4 = __ldg(cs + i4), s4 = __ldg(sn + i4);
                const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = 4 * i4 + e;
                  const float x = __uint_as_float(ra[i]) * rinv, y = __uint_as_float(rb[i]) * rinv;
                  a[i] = x * cv[e] - y * sv[e];
                  b[i] = y * cv[e] + x * sv[e];
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                a[i] = __uint_as_float(ra[i]) * rinv;
                b[i] = __uint_as_float(rb[i]) * rinv;
              }
            }
            __nv_bfloat16* dst;
            if (section == 0) {
              dst = args.q_out + (size_t)row * hd + head * 128;
            } else {
              const int sess = row / args.b.n_tok;
              const int j = row - sess * args.b.n_tok;
              const long long prow = args.b.base[sess] + args.b.valid[sess] + j;
              dst = (section == 1 ? args.k_layer : args.v_layer) + prow * hd + head * 128;
            }
            store_bf16x32(dst + half * 32, a);
            store_bf16x32(dst + 64 + half * 32, b);
          }
        }
      } else if (EPI == EPI_RESID) {
        float4* stg = reinterpret_cast<float4*>(smem + C::EPI_OFF) + quarter * (32 * 8);
        float ssq[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) ssq[it] = 0.f;
        // unrolled so the two residual buffers stay in registers
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          if (c + 1 < BN / 32) load_res(c + 1, res[(c + 1) & 1]);
          uint32_t r[32];
          tmem_ld32(tbase + c * 32, r);
          tmem_wait_ld(r);
          // row `lane` of the chunk; float4 slot k stored at k ^ (lane & 7) (no bank conflicts)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            stg[lane * 8 + (k ^ (lane & 7))] =
                make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                            __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
          __syncwarp();
          const int col = n0 + c * 32 + cg * 4;
          float gv[4] = {1.f, 1.f, 1.f, 1.f};
          if (args.g_next) {
            const uint2 gu = __ldg(reinterpret_cast<const uint2*>(args.g_next + col));
            const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gu.x));
            const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gu.y));
            gv[0] = g01.x; gv[1] = g01.y; gv[2] = g23.x; gv[3] = g23.y;
          }
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rl = 4 * it + rsub;
            const int rr = wrow0 + rl;
            const float4 a = stg[rl * 8 + (cg ^ (rl & 7))];
            if (rr >= args.M) continue;
            float4 x = res[c & 1][it];
            x.x += a.x;
            x.y += a.y;
            x.z += a.z;
            x.w += a.w;
            *reinterpret_cast<float4*>((float*)args.C + (size_t)rr * args.ldc + col) = x;
            if (args.g_next) {
              // the next RMSNorm's numerator bf16(x g) and this row's sum of squares
              ssq[it] = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, ssq[it]))));
              uint2 o;
              o.x = pack_bf16x2(x.x * gv[0], x.y * gv[1]);
              o.y = pack_bf16x2(x.z * gv[2], x.w * gv[3]);
              *reinterpret_cast<uint2*>(args.xg + (size_t)rr * args.ldc + col) = o;
            }
          }
          __syncwarp();   // the next chunk overwrites the transpose buffer
        }
        if (args.g_next) {
          // each row's partial sum over this tile: the 8 lanes of its column groups
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            float t = ssq[it];
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            t += __shfl_xor_sync(0xffffffffu, t, 4);
            const int rr = wrow0 + 4 * it + rsub;
            if (cg == 0 && rr < args.M) args.ss_out[(size_t)rr * args.ss_ld + n0 / BN] = t;
          }
        }
      } else if (EPI == EPI_SWIGLU) {
        // columns 128 b + [0, 64) of the tile are gate units, 128 b + [64, 128) their up
        // partners: out[(n0 + 128 b) / 2 + c] = silu(gate) * up, bf16
        for (int b = 0; b < BN / 128; ++b) {
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t rg[32], ru[32];
            tmem_ld32(tbase + b * 128 + hf * 32, rg);
            tmem_ld32(tbase + b * 128 + 64 + hf * 32, ru);
            tmem_wait_ld(rg);
            reg_fence(ru);
            if (!live) continue;
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float g = __uint_as_float(rg[i]) * rinv, u = __uint_as_float(ru[i]) * rinv;
              v[i] = g / (1.f + __expf(-g)) * u;
            }
            store_bf16x32((__nv_bfloat16*)args.C + (size_t)row * args.ldc + (n0 + b * 128) / 2 + hf * 32, v);
          }
        }
      } else {
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tbase + c * 32, r);
          tmem_wait_ld(r);
          if (!live) continue;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          const int col = n0 + c * 32;
          if (EPI == EPI_F32) {
            float4* d = reinterpret_cast<float4*>((float*)args.C + (size_t)sl * args.M * args.ldc +
                                                  (size_t)row * args.ldc + col);
#pragma unroll
            for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          } else {
            if (EPI == EPI_GELU) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = gelu_tanh(v[i] * rinv);
            }
            store_bf16x32((__nv_bfloat16*)args.C + (size_t)row * args.ldc + col, v);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
        else
          mbar_arrive(&acc_empty[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1u;
    }
  }

  // neither CTA of a pair frees its TMEM or exits while the pair's MMAs, loads or
  // remote arrivals may still touch it
  tc_fence_before();
  if (PAIR) {
    __syncwarp();
    cluster_sync();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int EPI, bool PAIR>
int launch_bn(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, int sms,
              cudaStream_t s) {
  using C = Cfg<BN, PAIR>;
  constexpr int TM = PAIR ? 2 * BM : BM;
  const int tiles = ((args.M + TM - 1) / TM) * (args.N / BN) * (args.k_splits > 1 ? args.k_splits : 1);
  const int units = PAIR ? sms / 2 : sms;
  const int grid = (tiles < units ? tiles : units) * (PAIR ? 2 : 1);
  auto kern = gemm_tc_kernel<BN, EPI, PAIR>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 1 : 0;
  return record_cuda(cudaLaunchKernelEx(&cfg, kern, a, b, args));
}

}  // namespace gtc

bool gemm_tc_pair(int M, int N, int hd, int epi, int sms) {
  // Pairs halve each SM's weight traffic but add a cross-SM hop to every stage;
  // they pay off when every pair has several tiles to pipeline (measured on the
  // 924-row projections: +4-5 % for N = 9216 and 12288 at 2-2.6 tiles per pair,
  // -6-8 % for N = 3072 at under one).
  if (M <= gtc::BM || sms < 2) return false;
  const int bn = gemm_tc_block_n(M, N, hd, epi, sms, true);
  if (!bn) return false;
  const long long tiles = (long long)((M + 2 * gtc::BM - 1) / (2 * gtc::BM)) * (N / bn);
  return 2 * tiles >= 3LL * (sms / 2);
}

int gemm_tc_block_n(int M, int N, int hd, int epi, int sms, bool pair) {
  // N-tile width minimising (waves of the persistent grid) x (time per tile); ties
  // go to the wider tile.  A tile's time is modelled as BN + 128 columns: a k-block's
  // time is set mostly by the round trip of its operand stages, not by BN (measured
  // per k-block on 924 / 7392-row projections: ~680 cycles for 256-wide pair tiles,
  // ~626 for 128-wide ones), so narrow tiles cost more per column.  The QKV epilogue
  // works on whole 128-wide heads.  Pairs take 256-row tiles and run on sms / 2 units.
  const int cands[3] = {256, 192, 128};
  if (pair) sms /= 2;
  const int tm = pair ? 2 * gtc::BM : gtc::BM;
  const long long m_tiles = (M + tm - 1) / tm;
  int best = 0;
  long long best_cost = 0;
  for (int bn : cands) {
    if (N % bn) continue;
    if (epi == EPI_QKV && (bn % 128 || hd % bn)) continue;
    if (epi == EPI_SWIGLU && bn % 128) continue;   // whole gate / up block pairs
    const long long tiles = m_tiles * (N / bn);
    const long long cost = ((tiles + sms - 1) / sms) * (bn + 128);
    if (!best || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

int gemm_tc_k_splits(int M, int N, int K, int block_n, int sms) {
  if (block_n <= 0 || N % block_n) return 1;
  const long long tiles = (long long)((M + gtc::BM - 1) / gtc::BM) * (N / block_n);
  if (2 * tiles > sms) return 1;
  long long sp = sms / tiles;
  const long long by_k = (K / gtc::BK) / 4;   // at least 4 k-blocks per slice
  if (sp > by_k) sp = by_k;
  if (sp > 16) sp = 16;
  return sp > 1 ? (int)sp : 1;
}

int launch_gemm_tc(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, int sms,
                   cudaStream_t s) {
  if (args.M <= 0) return SFM_OK;
  const bool pair = args.pair != 0;
  if (pair && sms < 2) return SFM_EUNSUPPORTED;
  const int bn = args.block_n;
  if (!bn || args.N % bn || args.K % gtc::BK || args.K <= 0) return SFM_EUNSUPPORTED;
  if (args.epi == EPI_QKV && (args.hd % bn || args.N != 3 * args.hd)) return SFM_EUNSUPPORTED;
  if (args.k_splits > 1 && (args.epi != EPI_F32 || pair || args.k_splits > args.K / gtc::BK))
    return SFM_EUNSUPPORTED;
#define SFM_GTC(BN_, E)                                                              \
  if (bn == BN_ && args.epi == E)                                                    \
    return pair ? gtc::launch_bn<BN_, E, true>(a, b, args, sms, s)                  \
                : gtc::launch_bn<BN_, E, false>(a, b, args, sms, s);
  SFM_GTC(256, EPI_F32)
  SFM_GTC(256, EPI_GELU)
  SFM_GTC(256, EPI_RESID)
  SFM_GTC(256, EPI_STORE)
  SFM_GTC(256, EPI_QKV)
  SFM_GTC(192, EPI_F32)
  SFM_GTC(192, EPI_GELU)
  SFM_GTC(192, EPI_RESID)
  SFM_GTC(192, EPI_STORE)
  SFM_GTC(128, EPI_F32)
  SFM_GTC(128, EPI_GELU)
  SFM_GTC(128, EPI_RESID)
  SFM_GTC(128, EPI_STORE)
  SFM_GTC(128, EPI_QKV)
  SFM_GTC(256, EPI_SWIGLU)
  SFM_GTC(128, EPI_SWIGLU)
#undef SFM_GTC
  return SFM_EINVAL;
}

}  // namespace sfm
