// Attention of the current unit on the 5th-generation tensor cores (tcgen05).
//
// The performer form of block-causal attention ("Wan-Streamer" v0.1 blog,
// §3.3): every query of the current unit sees every valid cached key and every
// key of the current unit, so O = softmax(Q K^T / sqrt(D)) V over one key
// range per session, D = 128.
//
// One CTA = one (session, head, 256-query block, key split): two 128-row
// query tiles A and B share every K/V tile.  Each session has its own split
// count; the CTAs are numbered session by session in a host-given order (longest
// CTAs first, so the SMs finish together), and within a session split, head,
// query block, the query block fastest: the CTAs that read the same K/V tiles
// start together.  320 threads:
//   warp 0      TMA producer: both Q tiles once; K tiles (128 keys x 128 dims)
//               in a 3-stage ring, V tiles in a 2-stage ring (128-byte swizzle)
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma, alternating tiles:
//                 S_t = Q_t K_j^T   (M=128, N=128 keys, K=128 dims), smem x smem
//                 O_t += P_t V_j    (M=128, N=128 dims, K=128 keys), P from TMEM,
//                                   V from smem as an MN-major operand
//               S_t of the next key tile is issued once O_t's P V has completed
//               (P_t aliases S_t in TMEM).
//   warps 2-5   softmax of tile A, warps 6-9 softmax of tile B (thread = query
//               row): one pass over the S row in TMEM computes
//               p = 2^(s scale - m) against the running max m; P is held in
//               registers and written back over S as packed bf16.  A row's max
//               can only have grown by more than 2^8 if its tile sum of p passed
//               2^8, so only then is the tile's exact max taken (a second pass
//               over S), and only when it did grow by more (decided per warp: the
//               TMEM accesses are collective) is O rescaled in TMEM and P
//               recomputed from S.  Final O / l written as bf16 (one split) or as
//               fp32 partials + log2-sum-exp.
// TMEM columns: tile A S/P [0,128) O [128,256); tile B S/P [256,384) O [384,512).
// The last, partial key tile is masked in S, and its V rows past the key range
// are zeroed in shared memory before P V, so rows outside the range never
// contribute (whatever they hold).
// Block-causal form (AttnDesc::unit_rows > 0, several query units over a shared
// prefix): a CTA walks the key tiles up to its last row's limit, and each
// softmax thread masks the logits past its own row's limit, so keys of later
// units are neither loaded by CTAs that cannot see them nor seen by rows that
// may not.  A row can then have no visible key in a whole split: its running
// max stays -inf, its partial is 0 with log-sum-exp -inf, and the merge gives
// it weight 0.
#include <math.h>

#include <algorithm>
#include <vector>

#include "attn.cuh"
#include "sm100.cuh"

namespace sfm {

using namespace sm100;

namespace atc {

constexpr int BQ = kAttnQBoxRows, QT = 2, BKV = kAttnKVBoxRows, D = 128;
static_assert(BQ == 128 && BKV == 128, "tile shapes fixed by the TMEM / shared-memory plan");
constexpr int ROWS = BQ * QT;               // query rows per CTA
constexpr int THREADS = 320;
constexpr int KST = 3, VST = 2;
constexpr int HALF = 128 * 64 * 2;          // one [128 rows][64 cols] bf16 swizzle tile: 16 KB
constexpr int TILE = 2 * HALF;              // [128][128] bf16: 32 KB
constexpr int OFF_Q = 0;                    // Q_A, Q_B
constexpr int OFF_K = OFF_Q + QT * TILE;
constexpr int OFF_V = OFF_K + KST * TILE;
constexpr int OFF_BAR = OFF_V + VST * TILE;      // 229376
constexpr int SMEM = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleLog2 = 8.0f;

struct Args {
  AttnDesc a;
  int H;
  int ns[kMaxBatch];           // key splits of each session (1: O written directly)
  int order[kMaxBatch];        // sessions in CTA order
  int qtiles;                  // 256-row query blocks per session
  float scale_log2;
  long long total_rows;
  int kv_row0;                 // row offset of this layer inside the K/V tensor maps
  __nv_bfloat16* o;            // [total_rows][H][D] (one split)
  float* o_part;               // [split][total_rows][H][D] (sessions of more than one split)
  float* lse_part;             // [split][total_rows][H]
  int* err;
  unsigned long long wait_ns;  // bound of every wait
  int fault;                   // SFM_FAULT_ATTN_NO_LOADS: the producer issues no loads (test only)
};

// 10 warps: two of the four SM sub-partitions hold three warps, which caps a
// thread at 16384 / (3 * 32) registers -- the launch bound makes ptxas respect it.
__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ Args args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;   // [QT]
  uint64_t* p_full = s_full + QT;     // [QT]
  uint64_t* o_done = p_full + QT;     // [QT]
  uint64_t* drain = o_done + QT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // the CTA's work, decoded once below: the softmax warps read it back from shared
  // memory where they need it, so that none of it holds registers through their key loop
  volatile int* cta_info = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int rem = blockIdx.x, sess = args.order[0];
  for (int i = 0; i < args.a.n; ++i) {
    sess = args.order[i];
    const int c = args.ns[sess] * args.H * args.qtiles;
    if (rem < c) break;
    rem -= c;
  }
  const int n_splits = args.ns[sess];
  const int qb = rem % args.qtiles;
  rem /= args.qtiles;
  const int h = rem % args.H, split = rem / args.H;
  const long long row0 = (long long)sess * args.a.rows_per + (long long)qb * ROWS;
  // keys of this CTA: up to the limit of its last query row (block-causal: the
  // rows' own limits are masked per row below)
  const int q_last = min(args.a.rows_per, qb * ROWS + ROWS) - 1;
  const int nkeys = attn_key_limit(args.a.nkeys[sess], args.a.rows_per, args.a.unit_rows, q_last);
  const long long kbase = args.a.kbase[sess];
  const int ntiles = (nkeys + BKV - 1) / BKV;
  const int tps = (ntiles + n_splits - 1) / n_splits;
  const int t0 = min(ntiles, split * tps);
  const int t1 = min(ntiles, t0 + tps);
  const int T = t1 - t0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < KST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);          // one arrival per softmax warp of the tile
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    cta_info[0] = h;
    cta_info[1] = split;
    cta_info[2] = n_splits;
    cta_info[3] = sess;
    cta_info[4] = qb;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&map_q);
    tma_prefetch(&map_k);
    tma_prefetch(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && T > 0 && !(args.fault & SFM_FAULT_ATTN_NO_LOADS)) {
      // ---------------- TMA producer ----------------
      int kp[KST], vp[VST];               // parity of the last load into each stage
      for (int i = 0; i < KST; ++i) kp[i] = -1;
      for (int i = 0; i < VST; ++i) vp[i] = -1;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, QT * TILE);
      for (int t = 0; t < QT; ++t) {
        tma_load_3d(base + OFF_Q + t * TILE, &map_q, q_full, 0, h, (int)(row0 + t * BQ));
        tma_load_3d(base + OFF_Q + t * TILE + HALF, &map_q, q_full, 64, h, (int)(row0 + t * BQ));
      }
      auto load_k = [&](int i) -> bool {   // i: tile index relative to t0
        const int s = i % KST;
        const uint32_t par = (uint32_t)((i / KST) & 1);
        if (!mbar_wait(&k_empty[s], par ^ 1u, abort, args.err, 0x201, args.wait_ns)) return false;
        const int krow = args.kv_row0 + (int)(kbase + (long long)(t0 + i) * BKV);
        mbar_arrive_expect_tx(&k_full[s], TILE);
        tma_load_3d(base + OFF_K + s * TILE, &map_k, &k_full[s], 0, h, krow);
        tma_load_3d(base + OFF_K + s * TILE + HALF, &map_k, &k_full[s], 64, h, krow);
        kp[s] = (int)par;
        return true;
      };
      auto load_v = [&](int i) -> bool {
        const int s = i % VST;
        const uint32_t par = (uint32_t)((i / VST) & 1);
        if (!mbar_wait(&v_empty[s], par ^ 1u, abort, args.err, 0x202, args.wait_ns)) return false;
        const int krow = args.kv_row0 + (int)(kbase + (long long)(t0 + i) * BKV);
        mbar_arrive_expect_tx(&v_full[s], TILE);
        tma_load_3d(base + OFF_V + s * TILE, &map_v, &v_full[s], 0, h, krow);
        tma_load_3d(base + OFF_V + s * TILE + HALF, &map_v, &v_full[s], 64, h, krow);
        vp[s] = (int)par;
        return true;
      };
      // order of need by the MMA issuer: S(0); then per j: P V (V_j), S(j+1) (K_{j+1})
      if (ok) ok = load_k(0);
      if (ok && T > 1) ok = load_k(1);
      for (int j = 0; j < T && ok; ++j) {
        ok = load_v(j);
        if (ok && j + 2 < T) ok = load_k(j + 2);
      }
      if (!ok) {   // unwinding: let issued loads land before the CTA exits
        mbar_drain(q_full, 0, args.wait_ns);
        for (int i = 0; i < KST; ++i)
          if (kp[i] >= 0) mbar_drain(&k_full[i], (uint32_t)kp[i], args.wait_ns);
        for (int i = 0; i < VST; ++i)
          if (vp[i] >= 0) mbar_drain(&v_full[i], (uint32_t)vp[i], args.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && T > 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(BQ, D, false, true);
      bool ok = mbar_wait(q_full, 0, abort, args.err, 0x203, args.wait_ns), issued = false;
      auto issue_s = [&](int t, int ks) {   // S_t = Q_t K^T from K stage ks
        const uint32_t qa = base + OFF_Q + t * TILE, ka = base + OFF_K + ks * TILE;
        const uint32_t d = tmem + (uint32_t)(t * 256);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t sub = (uint32_t)(kk >> 2) * HALF;
          const uint64_t da = sw128_desc(qa + sub, 16, 1024) + (uint64_t)(2 * (kk & 3));
          const uint64_t db = sw128_desc(ka + sub, 16, 1024) + (uint64_t)(2 * (kk & 3));
          umma_bf16(d, da, db, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
        issued = true;
      };
      if (ok && (ok = mbar_wait(&k_full[0], 0, abort, args.err, 0x204, args.wait_ns))) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&k_empty[0]);
      }
      // per key tile j: P_A V, S_A(j+1), P_B V, S_B(j+1) -- tile A never waits on tile B,
      // so the two softmax warpgroups run half a period apart
      for (int j = 0; j < T && ok; ++j) {
        const int vs = j % VST;
        const bool more = j + 1 < T;
        const int ks = (j + 1) % KST;
        if (!mbar_wait(&v_full[vs], (uint32_t)((j / VST) & 1), abort, args.err, 0x206, args.wait_ns)) {
          ok = false;
          break;
        }
        const uint32_t va = base + OFF_V + vs * TILE;
        for (int t = 0; t < QT && ok; ++t) {
          if (!mbar_wait(&p_full[t], (uint32_t)(j & 1), abort, args.err, 0x205, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pa = tmem + (uint32_t)(t * 256);          // P_t: packed bf16, 64 columns
          const uint32_t d = tmem + (uint32_t)(t * 256 + 128);     // O_t
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // V as MN-major B: 64-dim halves HALF bytes apart, 16 keys = 2048 B per K step
            const uint64_t db = sw128_desc(va + (uint32_t)kk * 2048u, HALF, 1024);
            umma_bf16_tmem_a(d, pa + (uint32_t)(kk * 8), db, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&o_done[t]);
          if (t == QT - 1) umma_commit(&v_empty[vs]);
          if (more) {
            if (t == 0 &&
                !mbar_wait(&k_full[ks], (uint32_t)(((j + 1) / KST) & 1), abort, args.err, 0x204, args.wait_ns)) {
              ok = false;
              break;
            }
            // S_t(j+1) overwrites P_t(j): wait until O_t's P V of this tile has completed
            if (!mbar_wait(&o_done[t], (uint32_t)(j & 1), abort, args.err, 0x20B, args.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t, ks);
            if (t == QT - 1) umma_commit(&k_empty[ks]);
          }
        }
      }
      if (!ok && issued) {
        umma_commit(drain);
        mbar_drain(drain, 0, args.wait_ns);
      }
    }
  } else {
    // ---------------- softmax + output (thread = query row of tile t) ----------------
    const int t = (warp - 2) >> 2;                        // 0: tile A, 1: tile B
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                    // row inside the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t col_s = (uint32_t)(t * 256), col_o = col_s + 128;
    const int q_rows = min(BQ, args.a.rows_per - qb * ROWS - t * BQ);   // may be <= 0
    // this row's key limit (rows past the session's end take the last row's)
    const int my_keys = attn_key_limit(args.a.nkeys[sess], args.a.rows_per, args.a.unit_rows,
                                       min(qb * ROWS + t * BQ + r, args.a.rows_per - 1));
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    const float sc = args.scale_log2;
    for (int j = 0; j < T && ok; ++j) {
      // the key limits of this tile do not depend on S: settled before waiting for it
      const int kvalid = nkeys - (t0 + j) * BKV;         // > 0; < BKV only on the last tile
      const int kmine = my_keys - (t0 + j) * BKV;        // this row's; may be <= 0
      const int kwarp = __reduce_min_sync(0xffffffffu, kmine);
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], (uint32_t)(j & 1), abort, args.err, 0x207, args.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (kwarp < BKV) {
        // partial tile for some row of the warp: overwrite the row's logits past its
        // key limit with -inf (the TMEM accesses are warp-collective)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c * 32 + 32 <= kwarp) continue;
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + col_s + c * 32, u);
          tmem_wait_ld(u);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= kmine) u[i] = __float_as_uint(-INFINITY);
          tmem_st32(tmem + lane_base + col_s + c * 32, u);
        }
        tmem_st_wait();
      }
      // P = 2^(s scale - m) with m the running row max.  From the second key tile on, one
      // pass over the S row computes P against the running max; the row's tile sum of P
      // bounds its growth (some p > 2^8 only if the sum passed 2^8), so the tile's exact
      // max is taken only then, and only when some row of the warp grows by more than
      // 2^8 is the attempt dropped: O is rescaled and P recomputed from S (still intact
      // in TMEM, as P is held in registers until the row is done).  The first tile takes
      // its max first.  Loads of the next 32-column chunk overlap work on the current one.
      uint32_t pk[4][16];
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      float mx = -INFINITY;
      bool fresh = j == 0;                                // P still to be computed
      if (!fresh) {
        // a row with no visible key so far (block-causal, a later split) has m = -inf:
        // its attempt below is dropped by the rescale test, so any finite base serves
        const float neg_m = m == -INFINITY ? 0.f : -m;
        uint32_t u[2][32];
        tmem_ld32(tmem + lane_base + col_s, u[0]);
        tmem_wait_ld(u[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld32(tmem + lane_base + col_s + (c + 1) * 32, u[(c + 1) & 1]);
          const float* sv = reinterpret_cast<const float*>(u[c & 1]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2_approx(fmaf(sv[2 * i], sc, neg_m));
            const float p1 = ex2_approx(fmaf(sv[2 * i + 1], sc, neg_m));
            l4[(2 * i) & 3] += p0;
            l4[(2 * i + 1) & 3] += p1;
            pk[c][i] = pack_bf16x2(p0, p1);
          }
          if (c + 1 < 4) tmem_wait_ld(u[(c + 1) & 1]);
        }
        // a row's max can only have grown by more than 2^8 if its tile sum of p passed 2^8
        // (every p > 0); only then is the tile's exact row max taken, from S (intact in TMEM)
        const float lt = (l4[0] + l4[1]) + (l4[2] + l4[3]);
        bool grown = false;
        if (__any_sync(0xffffffffu, !(lt <= 256.f))) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[32];
            tmem_ld32(tmem + lane_base + col_s + c * 32, w);
            tmem_wait_ld(w);
            const float* sv = reinterpret_cast<const float*>(w);
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              m4[0] = fmax3(m4[0], sv[i], sv[i + 1]);
              m4[1] = fmax3(m4[1], sv[i + 2], sv[i + 3]);
              m4[2] = fmax3(m4[2], sv[i + 4], sv[i + 5]);
              m4[3] = fmax3(m4[3], sv[i + 6], sv[i + 7]);
            }
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sc;
          grown = __any_sync(0xffffffffu, mx > m + kRescaleLog2);
        }
        if (grown) {
          // O_t's previous P V has completed (S_t(j) was issued after it): rescale it
          const float m_new = fmaxf(m, mx);
          const float alpha = m == -INFINITY ? 0.f : ex2_approx(m - m_new);   // O, l are 0 then
          l *= alpha;
          m = m_new;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + col_o + c * 32, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + col_o + c * 32, o);
          }
          fresh = true;
        }
      } else {
        // first tile: row max of the raw logits (the scale is positive)
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint32_t u[2][32];
        tmem_ld32(tmem + lane_base + col_s, u[0]);
        tmem_wait_ld(u[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld32(tmem + lane_base + col_s + (c + 1) * 32, u[(c + 1) & 1]);
          const float* sv = reinterpret_cast<const float*>(u[c & 1]);
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            m4[0] = fmax3(m4[0], sv[i], sv[i + 1]);
            m4[1] = fmax3(m4[1], sv[i + 2], sv[i + 3]);
            m4[2] = fmax3(m4[2], sv[i + 4], sv[i + 5]);
            m4[3] = fmax3(m4[3], sv[i + 6], sv[i + 7]);
          }
          if (c + 1 < 4) tmem_wait_ld(u[(c + 1) & 1]);
        }
        m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sc;
      }
      if (__any_sync(0xffffffffu, fresh)) {
        const float neg_m = m == -INFINITY ? 0.f : -m;   // every key of the row masked: p = 0
        l4[0] = l4[1] = l4[2] = l4[3] = 0.f;
        uint32_t u[2][32];
        tmem_ld32(tmem + lane_base + col_s, u[0]);
        tmem_wait_ld(u[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld32(tmem + lane_base + col_s + (c + 1) * 32, u[(c + 1) & 1]);
          const float* sv = reinterpret_cast<const float*>(u[c & 1]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2_approx(fmaf(sv[2 * i], sc, neg_m));
            const float p1 = ex2_approx(fmaf(sv[2 * i + 1], sc, neg_m));
            l4[(2 * i) & 3] += p0;
            l4[(2 * i + 1) & 3] += p1;
            pk[c][i] = pack_bf16x2(p0, p1);
          }
          if (c + 1 < 4) tmem_wait_ld(u[(c + 1) & 1]);
        }
      }
      // P as packed bf16 pairs over the S row: keys [32 c, 32 c + 32) -> columns [16 c, 16 c + 16)
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st16(tmem + lane_base + col_s + c * 16, pk[c]);
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      tmem_st_wait();
      if (t == 0 && kvalid < BKV) {
        // zero the V rows of the partial tile past the key range once the tile has
        // landed (tile A's warps; both P V products are issued after tile A's P is ready)
        const int vs = j % VST;
        if (!__all_sync(0xffffffffu, mbar_wait(&v_full[vs], (uint32_t)((j / VST) & 1), abort, args.err, 0x209, args.wait_ns))) {
          ok = false;
          break;
        }
        if (r >= kvalid) {
          uint4* v0 = reinterpret_cast<uint4*>(smem + OFF_V + vs * TILE + r * 128);
          uint4* v1 = reinterpret_cast<uint4*>(smem + OFF_V + vs * TILE + HALF + r * 128);
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            v0[q] = z;
            v1[q] = z;
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    // ---- output ----
    if (ok && T > 0) {
      if (!__all_sync(0xffffffffu, mbar_wait(&o_done[t], (uint32_t)((T - 1) & 1), abort, args.err, 0x20A, args.wait_ns))) ok = false;
      tc_fence_after();
    }
    const int h_o = cta_info[0], split_o = cta_info[1], n_splits_o = cta_info[2];
    const long long row0_o = (long long)cta_info[3] * args.a.rows_per + (long long)cta_info[4] * ROWS;
    const long long grow = row0_o + t * BQ + r;
    const long long ld = (long long)args.H * D;
    const bool have = ok && T > 0 && l > 0.f;
    const float inv = have ? 1.f / l : 0.f;
    if (ok) {
      // Stage the warp's 32 normalised rows in shared memory, then write whole rows
      // (one row per warp instruction: coalesced).  The staging area is the Q and K
      // stages: the last S MMA of both tiles was issued before this tile's last
      // P V, whose completion o_done signalled, so nothing reads them any more
      // (the other tile's last P V may still read a V stage, which stays untouched).
      // Row `lane` keeps its float4 slot q at q ^ lane: no bank conflicts either way.
      float4* stage = reinterpret_cast<float4*>(smem + OFF_Q) + (warp - 2) * (32 * 32);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        if (T > 0) {
          tmem_ld32(tmem + lane_base + col_o + c * 32, u);
          tmem_wait_ld(u);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 f;
          f.x = have ? __uint_as_float(u[4 * q]) * inv : 0.f;
          f.y = have ? __uint_as_float(u[4 * q + 1]) * inv : 0.f;
          f.z = have ? __uint_as_float(u[4 * q + 2]) * inv : 0.f;
          f.w = have ? __uint_as_float(u[4 * q + 3]) * inv : 0.f;
          stage[lane * 32 + ((c * 8 + q) ^ lane)] = f;
        }
      }
      __syncwarp();
      const long long grow0 = row0_o + t * BQ + quarter * 32;   // global row of the warp's lane 0
      for (int rr = 0; rr < 32; ++rr) {
        if (quarter * 32 + rr >= q_rows) break;               // warp-uniform
        const float4 f = stage[rr * 32 + (lane ^ rr)];        // columns 4 lane .. 4 lane + 3
        if (n_splits_o == 1) {
          uint2 b;
          b.x = pack_bf16x2(f.x, f.y);
          b.y = pack_bf16x2(f.z, f.w);
          *reinterpret_cast<uint2*>(args.o + (grow0 + rr) * ld + h_o * D + 4 * lane) = b;
        } else {
          *reinterpret_cast<float4*>(args.o_part + ((long long)split_o * args.total_rows + grow0 + rr) * ld +
                                     h_o * D + 4 * lane) = f;
        }
      }
    } else if (r < q_rows) {
      // unwinding after a timed-out wait (loads may still land in shared memory):
      // zeros, written directly
      for (int c = 0; c < 4; ++c) {
        if (n_splits_o == 1) {
          uint4* d = reinterpret_cast<uint4*>(args.o + grow * ld + h_o * D + c * 32);
          for (int q = 0; q < 4; ++q) d[q] = make_uint4(0u, 0u, 0u, 0u);
        } else {
          float4* d = reinterpret_cast<float4*>(args.o_part + ((long long)split_o * args.total_rows + grow) * ld +
                                                h_o * D + c * 32);
          for (int q = 0; q < 8; ++q) d[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    if (r < q_rows && n_splits_o > 1)
      args.lse_part[((long long)split_o * args.total_rows + grow) * args.H + h_o] =
          have ? m + log2f(l) : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace atc

// Split counts from a cost model of the kernel, in microseconds on a B200:
//   CTA time  = (key tiles of the CTA) x kStepUs + kCtaUs (set-up, output, hand-over),
//   merge     = its bytes (fp32 partials of every split read, bf16 O written) / kMergeBps.
// More splits fill the SMs and shorten the longest CTA; each split adds fixed cost and
// merge traffic.  Block-causal calls count each query block's own key tiles.
namespace {

constexpr double kStepUs = 2.0, kCtaUs = 5.0, kMergeBps = 4.0e6;   // bytes per microsecond

// key tiles of query block b of a session with `keys` keys
long long block_tiles(int rows_per, long long keys, int unit_rows, int b) {
  const int last = (b + 1) * atc::ROWS < rows_per ? (b + 1) * atc::ROWS - 1 : rows_per - 1;
  const long long lim = unit_rows > 0 && keys < (1LL << 31)
                            ? attn_key_limit((int)keys, rows_per, unit_rows, last)
                            : keys;
  return (lim + atc::BKV - 1) / atc::BKV;
}

double merge_us(double rows_heads, int s) {
  return s > 1 ? (s * rows_heads * (atc::D + 1) * 4.0 + rows_heads * atc::D * 2.0) / kMergeBps : 0.0;
}

// One split count for identical sessions: kernel = max(waves x mean CTA time, longest
// CTA time), waves = ceil(CTAs / SMs).  tiles_of(i): key tiles of query block i
// (i < n_blocks); every block runs n_heads CTAs per split; merge_rows = query rows x heads.
template <typename F>
int choose_splits(F tiles_of, int n_blocks, int n_heads, double merge_rows, int sms) {
  long long max_tiles = 0;
  for (int i = 0; i < n_blocks; ++i) max_tiles = tiles_of(i) > max_tiles ? tiles_of(i) : max_tiles;
  const long long ctas = (long long)n_blocks * n_heads;
  int best = 1;
  double best_us = 0.0;
  for (int s = 1; s <= kMaxSplits; ++s) {
    if (s > 1 && max_tiles / s < 2) break;
    double sum_t = 0.0, max_t = 0.0;
    for (int i = 0; i < n_blocks; ++i) {
      const double t = (double)((tiles_of(i) + s - 1) / s) * kStepUs + kCtaUs;
      sum_t += t;
      max_t = t > max_t ? t : max_t;
    }
    const long long work = ctas * s;
    const double waves = (double)((work + sms - 1) / sms);
    double us = waves * sum_t / n_blocks;
    if (max_t > us) us = max_t;
    us += merge_us(merge_rows, s);
    if (s == 1 || us < best_us) {
      best = s;
      best_us = us;
    }
  }
  return best;
}

// key tiles of CTA (split z of ns, query block b) of session i
long long cta_tiles(const AttnDesc& a, int i, int b, int ns, int z) {
  const long long t = block_tiles(a.rows_per, a.nkeys[i], a.unit_rows, b);
  const long long tps = (t + ns - 1) / ns;
  const long long t0 = z * tps < t ? z * tps : t;
  return (t0 + tps < t ? t0 + tps : t) - t0;
}

// The kernel's CTA order: sessions by the key tiles of their longest CTA, longest
// first (ties by index); within a session split, head, query block.
void cta_order(const AttnDesc& a, const int* ns, int* order) {
  const int qtiles = (a.rows_per + atc::ROWS - 1) / atc::ROWS;
  long long len[kMaxBatch];
  for (int i = 0; i < a.n; ++i) {
    len[i] = cta_tiles(a, i, qtiles - 1, ns[i], 0);   // the last block sees the most keys
    order[i] = i;
  }
  std::stable_sort(order, order + a.n, [&](int x, int y) { return len[x] > len[y]; });
}

// Kernel time of a per-session plan: its CTAs, in the kernel's order, each given to
// the SM that frees first (a binary min-heap of the SMs' finishing times).
double schedule_us(const AttnDesc& a, const int* ns, int n_heads, int sms, std::vector<double>& heap) {
  const int qtiles = (a.rows_per + atc::ROWS - 1) / atc::ROWS;
  int order[kMaxBatch];
  cta_order(a, ns, order);
  heap.assign((size_t)sms, 0.0);
  std::vector<double> len((size_t)qtiles);
  for (int k = 0; k < a.n; ++k) {
    const int i = order[k];
    for (int z = 0; z < ns[i]; ++z) {
      for (int b = 0; b < qtiles; ++b) len[b] = (double)cta_tiles(a, i, b, ns[i], z) * kStepUs + kCtaUs;
      for (int hh = 0; hh < n_heads; ++hh)
        for (int b = 0; b < qtiles; ++b) {
          // replace the root (earliest free SM) by its new finishing time and sift down
          const double v = heap[0] + len[b];
          size_t p = 0;
          for (;;) {
            size_t c = 2 * p + 1;
            if (c >= heap.size()) break;
            if (c + 1 < heap.size() && heap[c + 1] < heap[c]) ++c;
            if (heap[c] >= v) break;
            heap[p] = heap[c];
            p = c;
          }
          heap[p] = v;
        }
    }
  }
  double mk = 0.0;
  for (double t : heap) mk = t > mk ? t : mk;
  return mk;
}

}  // namespace

// n_sessions identical sessions of max_keys keys; block-causal calls (unit_rows > 0)
// count each query block's own key tiles.
int attention_tc_splits(int rows_per_session, int n_sessions, long long max_keys, int n_heads,
                        int sms, int unit_rows) {
  const int qtiles = (rows_per_session + atc::ROWS - 1) / atc::ROWS;
  return choose_splits(
      [&](int i) { return block_tiles(rows_per_session, max_keys, unit_rows, i % qtiles); },
      n_sessions * qtiles, n_heads, (double)n_sessions * rows_per_session * n_heads, sms);
}

// A batch whose sessions have their own key counts (ragged caches): a split count
// per session.  Candidates: one count for every session (1..kMaxSplits), and
// ns_i = ceil(T_i / L) (T_i: the tiles of session i's longest query block) for each
// CTA length L at which some session's count changes.  Each candidate is scored by
// list-scheduling its CTAs in the kernel's order (schedule_us) plus its merge; one
// whose lower bound -- max(total CTA time / SMs, longest CTA) + merge -- cannot beat
// the best scored so far is not scheduled.  A single session keeps the
// identical-sessions model.
int attention_tc_splits_batch(const AttnDesc& a, int n_heads, int sms, int* ns) {
  const int qtiles = (a.rows_per + atc::ROWS - 1) / atc::ROWS;
  if (a.n <= 1) {
    ns[0] = a.n == 1 ? attention_tc_splits(a.rows_per, 1, a.nkeys[0], n_heads, sms, a.unit_rows) : 1;
    return ns[0];
  }
  long long tmax[kMaxBatch], top = 0;
  for (int i = 0; i < a.n; ++i) {
    tmax[i] = block_tiles(a.rows_per, a.nkeys[i], a.unit_rows, qtiles - 1);
    top = tmax[i] > top ? tmax[i] : top;
  }
  struct Cand {
    int ns[kMaxBatch];
    double lb;
  };
  std::vector<Cand> cands;
  auto add = [&](const int* v) {
    for (const Cand& c : cands)
      if (std::equal(v, v + a.n, c.ns)) return;
    Cand c{};
    std::copy(v, v + a.n, c.ns);
    double total = 0.0, longest = 0.0, merge = 0.0;
    for (int i = 0; i < a.n; ++i) {
      for (int z = 0; z < v[i]; ++z)
        for (int b = 0; b < qtiles; ++b) {
          const double t = (double)cta_tiles(a, i, b, v[i], z) * kStepUs + kCtaUs;
          total += t * n_heads;
          longest = t > longest ? t : longest;
        }
      merge += merge_us((double)a.rows_per * n_heads, v[i]);
    }
    c.lb = (total / sms > longest ? total / sms : longest) + merge;
    cands.push_back(c);
  };
  int v[kMaxBatch];
  for (int s = 1; s <= kMaxSplits; ++s) {
    if (s > 1 && top / s < 2) break;
    for (int i = 0; i < a.n; ++i) v[i] = s;
    add(v);
  }
  std::vector<long long> lens;
  for (int i = 0; i < a.n; ++i)
    for (int s = 1; s <= kMaxSplits; ++s) lens.push_back((tmax[i] + s - 1) / s);
  std::sort(lens.begin(), lens.end());
  lens.erase(std::unique(lens.begin(), lens.end()), lens.end());
  for (long long L : lens) {
    if (L < 2) continue;
    for (int i = 0; i < a.n; ++i) {
      const long long s = (tmax[i] + L - 1) / L;
      v[i] = (int)(s < 1 ? 1 : s > kMaxSplits ? kMaxSplits : s);
    }
    add(v);
  }
  std::sort(cands.begin(), cands.end(), [](const Cand& x, const Cand& y) { return x.lb < y.lb; });
  std::vector<double> heap;
  const Cand* best = &cands[0];
  double best_us = -1.0;
  for (const Cand& c : cands) {
    if (best_us >= 0.0 && c.lb >= best_us) break;
    double us = schedule_us(a, c.ns, n_heads, sms, heap);
    for (int i = 0; i < a.n; ++i) us += merge_us((double)a.rows_per * n_heads, c.ns[i]);
    if (best_us < 0.0 || us < best_us) {
      best = &c;
      best_us = us;
    }
  }
  int mx = 1;
  for (int i = 0; i < a.n; ++i) {
    ns[i] = best->ns[i];
    mx = ns[i] > mx ? ns[i] : mx;
  }
  return mx;
}

// q: map over [rows][H][128]; k, v: maps over the key rows ([rows][H][128]).
int launch_attention_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const AttnDesc& a, int kv_row0, int n_heads, const int* ns, void* o,
                        float* o_part, float* lse_part, const Guard& gd, cudaStream_t s) {
  const long long total_rows = (long long)a.n * a.rows_per;
  if (total_rows == 0) return SFM_OK;
  atc::Args args{};
  args.a = a;
  args.H = n_heads;
  args.qtiles = (a.rows_per + atc::ROWS - 1) / atc::ROWS;
  int max_splits = 1;
  long long ctas = 0;
  for (int i = 0; i < a.n; ++i) {
    if (ns[i] < 1 || ns[i] > kMaxSplits) return SFM_EINVAL;
    args.ns[i] = ns[i];
    max_splits = ns[i] > max_splits ? ns[i] : max_splits;
    ctas += (long long)ns[i] * n_heads * args.qtiles;
  }
  cta_order(a, ns, args.order);
  args.scale_log2 = (float)(1.4426950408889634 / sqrt((double)atc::D));
  args.total_rows = total_rows;
  args.kv_row0 = kv_row0;
  args.o = (__nv_bfloat16*)o;
  args.o_part = o_part;
  args.lse_part = lse_part;
  args.err = gd.err;
  args.wait_ns = gd.wait_ns;
  args.fault = gd.fault;
  cudaFuncSetAttribute(atc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, atc::SMEM);
  int rc;
  {
    ProfScope ps(SFM_PROF_ATTN, s);
    atc::attn_tc_kernel<<<(unsigned)ctas, atc::THREADS, atc::SMEM, s>>>(mq, mk, mv, args);
    rc = record_cuda(cudaGetLastError());
  }
  if (rc || max_splits == 1) return rc;
  // one merge per split count > 1 among the sessions (one-split sessions are done)
  ProfScope ps(SFM_PROF_ATTN_MERGE, s);
  for (int c = 2; c <= max_splits && !rc; ++c) {
    MergeDesc md{};
    md.rows_per = a.rows_per;
    for (int i = 0; i < a.n; ++i)
      if (ns[i] == c) md.sess[md.n++] = i;
    if (md.n) rc = launch_attention_merge(o_part, lse_part, o, total_rows, n_heads, c, md, s);
  }
  return rc;
}

int launch_attention_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const AttnDesc& a, int kv_row0, int n_heads, int n_splits, void* o,
                        float* o_part, float* lse_part, const Guard& gd, cudaStream_t s) {
  int ns[kMaxBatch];
  for (int i = 0; i < kMaxBatch; ++i) ns[i] = n_splits;
  return launch_attention_tc(mq, mk, mv, a, kv_row0, n_heads, ns, o, o_part, lse_part, gd, s);
}

}  // namespace sfm
