// C ABI of libsfm: argument validation, ownership of the K/V pool and the
// scratch activations, session bookkeeping, and the per-step launch sequence
// of f_theta.  Every error is caught on the host before any launch.
#include <limits.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <new>

#include "attn.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "sm100.cuh"

using namespace sfm;

namespace {
// Error word of the standalone calls (sfm_attention*, sfm_linear): one per device
// that loads the library, like every file-scope device variable.
__device__ int g_call_err;
}  // namespace

namespace sfm {
static thread_local int g_last_cuda_error = 0;

int record_cuda(cudaError_t e) {
  count_launch();
  if (e == cudaSuccess) return SFM_OK;
  g_last_cuda_error = (int)e;
  return SFM_ECUDA;
}
}  // namespace sfm

struct sfm_handle {
  sfm_config cfg{};
  int n_tok = 0;
  int es = 2;                    // bytes per stored element
  int hd = 0;                    // H * D_h
  bool has_weights = false;
  const void *w_in = nullptr, *e_mod = nullptr, *g_final = nullptr, *w_out = nullptr;
  std::vector<const void*> g_attn, w_qkv, w_o, g_mlp, w_1, w_2;
  void* k_pool = nullptr;
  void* v_pool = nullptr;
  // solves run as one CUDA graph, captured on a private stream and updated in place
  bool graphs = true;
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t graph_exec[3] = {nullptr, nullptr, nullptr};   // plain / guided / units passes
  long long pool_used = 0;
  std::vector<Session> sessions;
  // scratch, sized for max_sessions * n_tok rows
  float* x = nullptr;        // [M][d] fp32 residual stream
  void* xn = nullptr;        // [M][d] normalised GEMM operand
  float* qkv32 = nullptr;    // [M][3 H D] fp32 projection output
  float* mlp32 = nullptr;    // [M][2F] fp32 gate / up projection (fp32 SwiGLU)
  void* q = nullptr;         // [M][H][D] rotated queries
  void* ao = nullptr;        // [M][H D] attention output
  void* hmlp = nullptr;      // [M][F] GELU(MLP-up)
  float* cos_t = nullptr;    // [M][D/2]
  float* ss = nullptr;       // [M][d / 128]: fused-RMSNorm partial sums of squares
  float* sin_t = nullptr;
  float* o_part = nullptr;   // [kMaxSplits][M][H][D]
  float* lse_part = nullptr; // [kMaxSplits][M][H]
  int* d_err = nullptr;      // device error word (bounded waits that timed out)
  volatile int* h_err = nullptr;   // pinned host copy of d_err, written at the end of each solve
  Guard gd;                  // d_err, wait bound and test-only faults of this handle's kernels
  int sms = 148;
  // TMA tensor maps (bf16 mode): activations over max_sessions * N rows, weights per layer
  CUtensorMap map_xn{}, map_ao{}, map_hmlp{};
  CUtensorMap map_q{}, map_kpool{}, map_vpool{};  // attention operands
  std::vector<CUtensorMap> map_wqkv, map_wo, map_w1, map_w2;
  int bn_qkv = 0, bn_o = 0, bn_up = 0, bn_down = 0;   // N-tile widths the weight maps use
  bool pair_qkv = false, pair_o = false, pair_up = false, pair_down = false;   // CTA pairs
  int ksplit_o = 1, ksplit_down = 1;     // K slices of the residual projections (few tiles)
  float* ws_splitk = nullptr;            // [slices][M][d] fp32 partials
  std::vector<void*> owned;

  void* layer_k(int l) const { return (char*)k_pool + (size_t)l * cfg.pool_tokens * hd * es; }
  void* layer_v(int l) const { return (char*)v_pool + (size_t)l * cfg.pool_tokens * hd * es; }
};

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int validate_config(const sfm_config* c) {
  if (!c) return SFM_EINVAL;
  if (c->n_layers < 1 || c->d_model < 1 || c->n_heads < 1 || c->head_dim < 1 || c->d_mlp < 1 ||
      c->c_lat < 1 || c->n_video < 0 || c->n_audio < 0 || c->n_video + c->n_audio < 1 ||
      c->unit_kv_tokens < 1 || c->max_sessions < 1 || c->pool_tokens < 0)
    return SFM_EINVAL;
  if (c->dtype != SFM_DTYPE_BF16 && c->dtype != SFM_DTYPE_FP32) return SFM_EINVAL;
  if (c->mlp != SFM_MLP_GELU && c->mlp != SFM_MLP_SWIGLU) return SFM_EINVAL;
  if (c->rope != SFM_ROPE_1D && c->rope != SFM_ROPE_3D) return SFM_EINVAL;
  if (c->rope == SFM_ROPE_3D && (c->grid_w < 1 || c->head_dim < 6)) return SFM_EINVAL;
  if (c->mlp == SFM_MLP_SWIGLU && c->d_mlp % 64) return SFM_EUNSUPPORTED;
  if (!(c->rms_eps >= 0.0) || !(c->rope_theta > 0.0)) return SFM_EINVAL;
  if (c->max_sessions > kMaxBatch) return SFM_EUNSUPPORTED;
  if ((long long)c->n_layers * c->pool_tokens >= (1LL << 31)) return SFM_EUNSUPPORTED;
  if (c->c_lat > 64 || c->d_model % 2 || c->d_model > 8192) return SFM_EUNSUPPORTED;
  const int hd = c->n_heads * c->head_dim;
  if (c->dtype == SFM_DTYPE_BF16) {
    // GEMM tiles: N in multiples of 128, K in multiples of 64; flash tiles: D_h = 128
    if (c->head_dim != 128 || c->d_model % 128 || c->d_mlp % 128 || (3 * hd) % 128 || hd % 64)
      return SFM_EUNSUPPORTED;
  } else {
    if (c->head_dim % 32 || c->head_dim > 128 || c->d_model % 64 || c->d_mlp % 64 ||
        (3 * hd) % 64 || hd % 16)
      return SFM_EUNSUPPORTED;
  }
  return SFM_OK;
}

template <typename T>
int dalloc(sfm_handle* h, T** p, size_t bytes) {
  void* q = nullptr;
  if (bytes == 0) bytes = 16;
  if (cudaMalloc(&q, bytes) != cudaSuccess) {
    cudaGetLastError();
    return SFM_ENOMEM;
  }
  h->owned.push_back(q);
  *p = (T*)q;
  return SFM_OK;
}

int session_ok(const sfm_handle* h, int s) {
  if (!h) return SFM_EINVAL;
  if (s < 0 || s >= (int)h->sessions.size() || !h->sessions[s].open) return SFM_ESESSION;
  return SFM_OK;
}

long long valid_tokens(const sfm_handle* h, const Session& s) {
  const long long u = s.units < s.cache_units ? s.units : s.cache_units;
  return u * h->cfg.unit_kv_tokens;
}

int fill_batch(const sfm_handle* h, int n, const int* sessions, BatchDesc* b) {
  memset(b, 0, sizeof(*b));
  b->n = n;
  b->n_tok = h->n_tok;
  b->n_video = h->cfg.n_video;
  for (int i = 0; i < n; ++i) {
    const Session& s = h->sessions[sessions[i]];
    b->base[i] = s.base_row;
    b->valid[i] = (int)valid_tokens(h, s);
    b->p0[i] = s.units * h->cfg.unit_kv_tokens;
    b->t_unit[i] = s.units;
  }
  return SFM_OK;
}

AttnDesc attn_desc(const BatchDesc& b) {
  AttnDesc a{};
  a.n = b.n;
  a.rows_per = b.n_tok;
  for (int i = 0; i < b.n; ++i) {
    a.kbase[i] = b.base[i];
    a.nkeys[i] = b.valid[i] + b.n_tok;
  }
  return a;
}

int make_a_map(CUtensorMap* m, const void* p, long long rows, int k) {
  const uint64_t dims[2] = {(uint64_t)k, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)k * 2};
  const uint32_t box[2] = {64, 128};
  return make_tmap_bf16(m, p, 2, dims, strides, box);
}

int make_b_map(CUtensorMap* m, const void* p, int n, int k, int block_n) {
  const uint64_t dims[2] = {(uint64_t)k, (uint64_t)n};
  const uint64_t strides[1] = {(uint64_t)k * 2};
  const uint32_t box[2] = {64, (uint32_t)block_n};
  return make_tmap_bf16(m, p, 2, dims, strides, box);
}

// rows of [rows][H][128] bf16 (queries, or keys / values), box box_rows x 64 dims of one head
int make_rows_map(CUtensorMap* m, const void* p, long long rows, int heads, int box_rows) {
  const uint64_t dims[3] = {128, (uint64_t)heads, (uint64_t)rows};
  const uint64_t strides[2] = {256, (uint64_t)heads * 256};
  const uint32_t box[3] = {64, 1, (uint32_t)box_rows};
  return make_tmap_bf16(m, p, 3, dims, strides, box);
}

GemmArgs gemm_args(int M, int N, int K, int epi, void* C, int ldc, const Guard& gd, int block_n,
                   bool pair) {
  GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.epi = epi;
  g.C = C;
  g.ldc = ldc;
  g.err = gd.err;
  g.wait_ns = gd.wait_ns;
  g.fault = gd.fault;
  g.hd = 0;
  g.block_n = block_n;
  g.pair = pair ? 1 : 0;
  return g;
}

struct Guidance {
  bool on = false;
  float scale = 1.f;
};

// One Euler step of f_theta for the sessions in b (RoPE table already filled).
// Guided: entries 2p, 2p + 1 are a conditional / unconditional pair sharing z[2p].
int run_step(sfm_handle* h, const BatchDesc& b, const AttnDesc& ad, float* const* z,
             float tau_from, float tau_to, float* const* v_out, const Guidance& gd,
             cudaStream_t s) {
  const sfm_config& c = h->cfg;
  const int M = b.n * b.n_tok;
  const int d = c.d_model, hd = h->hd, F = c.d_mlp, dt = c.dtype;
  const float eps = (float)c.rms_eps;
  int rc;
#define SFM_TRY(call)                \
  do {                               \
    if ((rc = (call)) != SFM_OK) return rc; \
  } while (0)
  const bool tc = dt == SFM_DTYPE_BF16;
  // bf16 path: every RMSNorm before a projection is split between the kernel that
  // last updates x (it writes bf16(x g) and per-tile sums of squares) and the
  // projection's epilogue (it scales each row by 1 / rms)
  const int ss_ld = (d + 127) / 128;
  int ss_n = ss_ld;                 // partial sums per row left by the last producer
  {
    ProfScope ps(SFM_PROF_ROWOPS, s);
    if (tc)
      SFM_TRY(launch_embed(b, z, h->w_in, h->e_mod, tau_from, h->x, d, c.c_lat, dt, s,
                           h->g_attn[0], h->xn, h->ss, ss_ld));
    else
      SFM_TRY(launch_embed(b, z, h->w_in, h->e_mod, tau_from, h->x, d, c.c_lat, dt, s));
  }
  auto normed = [&](GemmArgs g) {   // a consumer of the fused norm
    g.ss_in = h->ss;
    g.ss_n = ss_n;
    g.ss_ld = ss_ld;
    g.norm_d = d;
    g.norm_eps = eps;
    return g;
  };
  // a residual projection in K slices: fp32 partials, then x += their sum (and the
  // next norm's numerator and the row's whole sum of squares)
  auto resid_split = [&](const CUtensorMap& ma, const CUtensorMap& mb, int K, int bn, int slices,
                         const void* gain) {
    GemmArgs g = gemm_args(M, d, K, EPI_F32, h->ws_splitk, d, h->gd, bn, false);
    g.k_splits = slices;
    int r = launch_gemm_tc(ma, mb, g, h->sms, s);
    if (!r)
      r = launch_resid_splitk(h->x, h->ws_splitk, slices, M, d, gain, h->xn, h->ss, ss_ld, s);
    if (gain) ss_n = 1;
    return r;
  };
  auto norm_next = [&](GemmArgs g, const void* gain, int bn) {   // a producer
    if (!gain) return g;
    g.g_next = (const __nv_bfloat16*)gain;
    g.xg = (__nv_bfloat16*)h->xn;
    g.ss_out = h->ss;
    g.ss_ld = ss_ld;
    ss_n = d / bn;
    return g;
  };
  int splits[kMaxBatch];   // key splits of each session's attention
  if (tc) attention_tc_splits_batch(ad, c.n_heads, h->sms, splits);
  for (int l = 0; l < c.n_layers; ++l) {
    if (!tc) {
      ProfScope ps(SFM_PROF_ROWOPS, s);
      SFM_TRY(launch_rmsnorm(h->x, h->g_attn[l], h->xn, M, d, eps, dt, s));
    }
    if (tc) {
      // QKV projection with the norm's 1 / rms, RoPE and the cache-tail scatter fused in
      // the epilogue
      ProfScope ps(SFM_PROF_GEMM_QKV, s);
      GemmArgs g = normed(gemm_args(M, 3 * hd, d, EPI_QKV, nullptr, 0, h->gd, h->bn_qkv, h->pair_qkv));
      g.cos_t = h->cos_t;
      g.sin_t = h->sin_t;
      g.q_out = (__nv_bfloat16*)h->q;
      g.k_layer = (__nv_bfloat16*)h->layer_k(l);
      g.v_layer = (__nv_bfloat16*)h->layer_v(l);
      g.hd = hd;
      g.b = b;
      SFM_TRY(launch_gemm_tc(h->map_xn, h->map_wqkv[l], g, h->sms, s));
    } else {
      {
        ProfScope ps(SFM_PROF_GEMM_QKV, s);
        SFM_TRY(launch_gemm(h->xn, h->w_qkv[l], h->qkv32, M, 3 * hd, d, EPI_F32, dt, s));
      }
      ProfScope ps(SFM_PROF_ROWOPS, s);
      SFM_TRY(launch_rope_scatter(b, h->qkv32, h->cos_t, h->sin_t, h->q, h->layer_k(l),
                                  h->layer_v(l), c.n_heads, c.head_dim, dt, s));
    }
    if (tc) {
      SFM_TRY(launch_attention_tc(h->map_q, h->map_kpool, h->map_vpool, ad,
                                  (int)((long long)l * c.pool_tokens), c.n_heads, splits, h->ao,
                                  h->o_part, h->lse_part, h->gd, s));
    } else {
      SFM_TRY(launch_attention(ad, h->q, h->layer_k(l), h->layer_v(l), h->ao, c.n_heads,
                               c.head_dim, dt, 1, h->o_part, h->lse_part, s));
    }
    {
      ProfScope ps(SFM_PROF_GEMM_O, s);
      if (tc && h->ksplit_o > 1) {
        SFM_TRY(resid_split(h->map_ao, h->map_wo[l], hd, h->bn_o, h->ksplit_o, h->g_mlp[l]));
      } else if (tc) {
        SFM_TRY(launch_gemm_tc(h->map_ao, h->map_wo[l],
                               norm_next(gemm_args(M, d, hd, EPI_RESID, h->x, d, h->gd, h->bn_o, h->pair_o),
                                         h->g_mlp[l], h->bn_o),
                               h->sms, s));
      } else {
        SFM_TRY(launch_gemm(h->ao, h->w_o[l], h->x, M, d, hd, EPI_RESID, dt, s));
      }
    }
    if (!tc) {
      ProfScope ps(SFM_PROF_ROWOPS, s);
      SFM_TRY(launch_rmsnorm(h->x, h->g_mlp[l], h->xn, M, d, eps, dt, s));
    }
    {
      ProfScope ps(SFM_PROF_GEMM_UP, s);
      const bool swiglu = c.mlp == SFM_MLP_SWIGLU;
      if (tc) {
        SFM_TRY(launch_gemm_tc(h->map_xn, h->map_w1[l],
                               normed(gemm_args(M, swiglu ? 2 * F : F, d, swiglu ? EPI_SWIGLU : EPI_GELU,
                                                h->hmlp, F, h->gd, h->bn_up, h->pair_up)),
                               h->sms, s));
      } else if (swiglu) {
        SFM_TRY(launch_gemm(h->xn, h->w_1[l], h->mlp32, M, 2 * F, d, EPI_F32, dt, s));
        SFM_TRY(launch_swiglu(h->mlp32, h->hmlp, M, F, dt, s));
      } else {
        SFM_TRY(launch_gemm(h->xn, h->w_1[l], h->hmlp, M, F, d, EPI_GELU, dt, s));
      }
    }
    {
      ProfScope ps(SFM_PROF_GEMM_DOWN, s);
      if (tc && h->ksplit_down > 1) {
        SFM_TRY(resid_split(h->map_hmlp, h->map_w2[l], F, h->bn_down, h->ksplit_down,
                            l + 1 < c.n_layers ? h->g_attn[l + 1] : nullptr));
      } else if (tc) {
        SFM_TRY(launch_gemm_tc(h->map_hmlp, h->map_w2[l],
                               norm_next(gemm_args(M, d, F, EPI_RESID, h->x, d, h->gd, h->bn_down, h->pair_down),
                                         l + 1 < c.n_layers ? h->g_attn[l + 1] : nullptr, h->bn_down),
                               h->sms, s));
      } else {
        SFM_TRY(launch_gemm(h->hmlp, h->w_2[l], h->x, M, d, F, EPI_RESID, dt, s));
      }
    }
  }
  {
    ProfScope ps(SFM_PROF_HEAD, s);
    SFM_TRY(launch_head_euler(b, h->x, h->g_final, h->w_out, z, v_out, tau_to - tau_from, d,
                              c.c_lat, eps, dt, s, gd.on, gd.scale));
  }
#undef SFM_TRY
  return SFM_OK;
}

// The device error word goes to pinned host memory at the end of every solve, so
// a later call can refuse (SFM_EDEVICE) without synchronising.
int error_to_host(sfm_handle* h, cudaStream_t s) {
  if (!h->h_err) return SFM_OK;
  const cudaError_t e =
      cudaMemcpyAsync((void*)h->h_err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) return SFM_OK;
  g_last_cuda_error = (int)e;
  return SFM_ECUDA;
}

// SFM_EDEVICE once a solve's copy of the error word has reported a timed-out wait.
int device_error_pending(const sfm_handle* h) {
  return h->h_err && *h->h_err ? SFM_EDEVICE : SFM_OK;
}

int check_taus(const float* taus, int n_taus) {
  if (!taus || n_taus < 2) return SFM_EINVAL;
  for (int i = 0; i < n_taus; ++i)
    if (!isfinite(taus[i])) return SFM_EINVAL;
  return SFM_OK;
}

// The batch of one pass of f_theta and the attention over it: the sessions of a
// (batched, guided) solve, each seeing its whole cache and unit; or several units
// of one session under the general block-causal mask.
struct Pass {
  BatchDesc b;
  AttnDesc a;
};

int solve_direct(sfm_handle* h, const Pass& ps, float* const* z, const float* taus, int n_taus,
                 float* const* v_out, const Guidance& gd, cudaStream_t s) {
  int rc;
  {
    ProfScope prof(SFM_PROF_ROWOPS, s);
    rc = launch_rope_table(ps.b, h->cos_t, h->sin_t, h->cfg.head_dim, h->cfg.rope_theta, s,
                           h->cfg.rope == SFM_ROPE_3D, h->cfg.grid_w);
  }
  if (rc) return rc;
  for (int i = 0; i + 1 < n_taus; ++i) {
    rc = run_step(h, ps.b, ps.a, z, taus[i], taus[i + 1], v_out, gd, s);
    if (rc) return rc;
  }
  return error_to_host(h, s);
}

// A solve is several hundred small launches (8 per layer per Euler step).  They
// are captured into a graph on the handle's private stream and the graph is
// launched on the caller's stream; the executable graph is kept and updated in
// place from each new capture (same topology, new kernel arguments: positions,
// cache lengths, latent pointers), so repeated units pay neither instantiation
// nor per-launch overheads.  The profiler brackets every launch with events,
// so a profiled call launches directly.
int solve_pass(sfm_handle* h, const Pass& ps, float* const* z, const float* taus, int n_taus,
               float* const* v_out, cudaStream_t s, const Guidance& gd, int kind) {
  if (!h->graphs || !h->cap_stream || profiling_active())
    return solve_direct(h, ps, z, taus, n_taus, v_out, gd, s);
  cudaGraphExec_t& exec = h->graph_exec[kind];
  if (cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return record_cuda(cudaGetLastError());
  const int rc = solve_direct(h, ps, z, taus, n_taus, v_out, gd, h->cap_stream);
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(h->cap_stream, &g);
  if (rc || ec != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return rc ? rc : record_cuda(ec != cudaSuccess ? ec : cudaErrorStreamCaptureInvalidated);
  }
  if (exec) {
    cudaGraphExecUpdateResultInfo info;
    if (cudaGraphExecUpdate(exec, g, &info) != cudaSuccess) {
      cudaGetLastError();
      cudaGraphExecDestroy(exec);
      exec = nullptr;
    }
  }
  cudaError_t e = cudaSuccess;
  if (!exec) e = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) {
    exec = nullptr;
    return record_cuda(e);
  }
  return record_cuda(cudaGraphLaunch(exec, s));
}

// Graph slots of the three kinds of pass (different kernels, so each keeps its own
// executable graph and alternating them costs no re-instantiation).
constexpr int kGraphPlain = 0, kGraphGuided = 1, kGraphUnits = 2;

int solve(sfm_handle* h, int n, const int* sessions, float* const* z, const float* taus,
          int n_taus, float* const* v_out, cudaStream_t s, const Guidance& gd = Guidance{}) {
  Pass ps;
  fill_batch(h, n, sessions, &ps.b);
  ps.a = attn_desc(ps.b);
  return solve_pass(h, ps, z, taus, n_taus, v_out, s, gd, gd.on ? kGraphGuided : kGraphPlain);
}

}  // namespace

extern "C" {

int sfm_create(const sfm_config* cfg, const sfm_weights* w, sfm_handle** out) {
  if (!out) return SFM_EINVAL;
  *out = nullptr;
  int rc = validate_config(cfg);
  if (rc) return rc;
  sfm_handle* h = new (std::nothrow) sfm_handle();
  if (!h) return SFM_ENOMEM;
  h->cfg = *cfg;
  h->n_tok = cfg->n_video + cfg->n_audio;
  h->es = cfg->dtype == SFM_DTYPE_BF16 ? 2 : 4;
  h->hd = cfg->n_heads * cfg->head_dim;
  if (((long long)h->hd * h->es) % 16) {
    delete h;
    return SFM_EUNSUPPORTED;
  }
  if (w) {
    const void* const* arrays[6] = {w->g_attn, w->w_qkv, w->w_o, w->g_mlp, w->w_1, w->w_2};
    if (!aligned16(w->w_in) || !aligned16(w->e_mod) || !aligned16(w->g_final) ||
        !aligned16(w->w_out) || !w->w_in || !w->e_mod || !w->g_final || !w->w_out)
      rc = SFM_EINVAL;
    for (int a = 0; a < 6 && !rc; ++a) {
      if (!arrays[a]) rc = SFM_EINVAL;
      for (int l = 0; l < cfg->n_layers && !rc; ++l)
        if (!arrays[a][l] || !aligned16(arrays[a][l])) rc = SFM_EINVAL;
    }
    if (rc) {
      delete h;
      return rc;
    }
    h->has_weights = true;
    h->w_in = w->w_in;
    h->e_mod = w->e_mod;
    h->g_final = w->g_final;
    h->w_out = w->w_out;
    h->g_attn.assign(w->g_attn, w->g_attn + cfg->n_layers);
    h->w_qkv.assign(w->w_qkv, w->w_qkv + cfg->n_layers);
    h->w_o.assign(w->w_o, w->w_o + cfg->n_layers);
    h->g_mlp.assign(w->g_mlp, w->g_mlp + cfg->n_layers);
    h->w_1.assign(w->w_1, w->w_1 + cfg->n_layers);
    h->w_2.assign(w->w_2, w->w_2 + cfg->n_layers);
  }
  h->sessions.resize(cfg->max_sessions);
  const size_t L = cfg->n_layers, es = h->es, hd = h->hd;
  const size_t M = (size_t)cfg->max_sessions * h->n_tok;
  const size_t d = cfg->d_model, F = cfg->d_mlp;
  const size_t pool_bytes = L * (size_t)cfg->pool_tokens * hd * es;
  rc = dalloc(h, &h->k_pool, pool_bytes);
  if (!rc) rc = dalloc(h, &h->v_pool, pool_bytes);
  if (!rc && h->has_weights) {
    if (!rc) rc = dalloc(h, &h->x, M * d * 4);
    if (!rc) rc = dalloc(h, &h->xn, M * d * es);
    if (!rc) rc = dalloc(h, &h->qkv32, M * 3 * hd * 4);
    if (!rc) rc = dalloc(h, &h->q, M * hd * es);
    if (!rc) rc = dalloc(h, &h->ao, M * hd * es);
    if (!rc) rc = dalloc(h, &h->hmlp, M * F * es);
    if (!rc && cfg->mlp == SFM_MLP_SWIGLU && cfg->dtype == SFM_DTYPE_FP32)
      rc = dalloc(h, &h->mlp32, M * 2 * F * 4);
    if (!rc) rc = dalloc(h, &h->cos_t, M * (cfg->head_dim / 2) * 4);
    if (!rc) rc = dalloc(h, &h->ss, M * ((cfg->d_model + 127) / 128) * 4);
    if (!rc) rc = dalloc(h, &h->sin_t, M * (cfg->head_dim / 2) * 4);
    if (!rc && cfg->dtype == SFM_DTYPE_BF16) {
      rc = dalloc(h, &h->o_part, (size_t)kMaxSplits * M * hd * 4);
      if (!rc) rc = dalloc(h, &h->lse_part, (size_t)kMaxSplits * M * cfg->n_heads * 4);
    }
  }
  if (!rc) rc = dalloc(h, &h->d_err, sizeof(int));
  if (!rc) {
    void* hp = nullptr;
    if (cudaHostAlloc(&hp, sizeof(int), cudaHostAllocDefault) != cudaSuccess) {
      cudaGetLastError();
      rc = SFM_ENOMEM;
    } else {
      h->h_err = (volatile int*)hp;
      *h->h_err = 0;
    }
    h->gd.err = h->d_err;
  }
  // Zero everything once: rows a tile reads past a session's valid range must hold
  // finite values, never uninitialised bit patterns.
  if (!rc) {
    if (cudaMemset(h->k_pool, 0, pool_bytes) != cudaSuccess ||
        cudaMemset(h->v_pool, 0, pool_bytes) != cudaSuccess ||
        cudaMemset(h->d_err, 0, sizeof(int)) != cudaSuccess)
      rc = record_cuda(cudaGetLastError());
    if (!rc && h->has_weights &&
        (cudaMemset(h->xn, 0, M * d * es) != cudaSuccess ||
         cudaMemset(h->q, 0, M * hd * es) != cudaSuccess ||
         cudaMemset(h->ao, 0, M * hd * es) != cudaSuccess ||
         cudaMemset(h->hmlp, 0, M * F * es) != cudaSuccess))
      rc = record_cuda(cudaGetLastError());
  }
  if (!rc) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev);
    // a handle without its capture stream still works, with direct launches
    if (cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      h->cap_stream = nullptr;
    }
  }
  if (!rc && h->has_weights && cfg->dtype == SFM_DTYPE_BF16) {
    const int L_ = cfg->n_layers, d_ = cfg->d_model, hd_ = h->hd, F_ = cfg->d_mlp;
    rc = make_a_map(&h->map_xn, h->xn, (long long)M, d_);
    if (!rc) rc = make_rows_map(&h->map_q, h->q, (long long)M, cfg->n_heads, kAttnQBoxRows);
    if (!rc && cfg->pool_tokens > 0)
      rc = make_rows_map(&h->map_kpool, h->k_pool, (long long)L_ * cfg->pool_tokens, cfg->n_heads,
                         kAttnKVBoxRows);
    if (!rc && cfg->pool_tokens > 0)
      rc = make_rows_map(&h->map_vpool, h->v_pool, (long long)L_ * cfg->pool_tokens, cfg->n_heads,
                         kAttnKVBoxRows);
    if (!rc) rc = make_a_map(&h->map_ao, h->ao, (long long)M, hd_);
    if (!rc) rc = make_a_map(&h->map_hmlp, h->hmlp, (long long)M, F_);
    h->map_wqkv.resize(L_);
    h->map_wo.resize(L_);
    h->map_w1.resize(L_);
    h->map_w2.resize(L_);
    // mode and tile widths chosen for a full batch (max_sessions units); the weight
    // maps' boxes depend on both
    const int mm = (int)M;
    h->pair_qkv = gemm_tc_pair(mm, 3 * hd_, hd_, EPI_QKV, h->sms);
    h->pair_o = gemm_tc_pair(mm, d_, 0, EPI_RESID, h->sms);
    const bool swiglu = cfg->mlp == SFM_MLP_SWIGLU;
    const int up_n = swiglu ? 2 * F_ : F_, up_epi = swiglu ? EPI_SWIGLU : EPI_GELU;
    h->pair_up = gemm_tc_pair(mm, up_n, 0, up_epi, h->sms);
    h->pair_down = gemm_tc_pair(mm, d_, 0, EPI_RESID, h->sms);
    h->bn_qkv = gemm_tc_block_n(mm, 3 * hd_, hd_, EPI_QKV, h->sms, h->pair_qkv);
    h->bn_o = gemm_tc_block_n(mm, d_, 0, EPI_RESID, h->sms, h->pair_o);
    h->bn_up = gemm_tc_block_n(mm, up_n, 0, up_epi, h->sms, h->pair_up);
    h->bn_down = gemm_tc_block_n(mm, d_, 0, EPI_RESID, h->sms, h->pair_down);
    if (!h->bn_qkv || !h->bn_o || !h->bn_up || !h->bn_down) rc = SFM_EUNSUPPORTED;
    if (!rc) {
      // split-K for residual projections whose tiles fill under half of the SMs
      if (!h->pair_o) h->ksplit_o = gemm_tc_k_splits(mm, d_, hd_, h->bn_o, h->sms);
      if (!h->pair_down) h->ksplit_down = gemm_tc_k_splits(mm, d_, F_, h->bn_down, h->sms);
      const int ks = h->ksplit_o > h->ksplit_down ? h->ksplit_o : h->ksplit_down;
      if (ks > 1) rc = dalloc(h, &h->ws_splitk, (size_t)ks * M * d_ * 4);
    }
    // the B box holds the weight rows one CTA stages: half the tile on pairs
    for (int l = 0; l < L_ && !rc; ++l) {
      rc = make_b_map(&h->map_wqkv[l], h->w_qkv[l], 3 * hd_, d_, h->bn_qkv / (h->pair_qkv ? 2 : 1));
      if (!rc) rc = make_b_map(&h->map_wo[l], h->w_o[l], d_, hd_, h->bn_o / (h->pair_o ? 2 : 1));
      if (!rc) rc = make_b_map(&h->map_w1[l], h->w_1[l], up_n, d_, h->bn_up / (h->pair_up ? 2 : 1));
      if (!rc) rc = make_b_map(&h->map_w2[l], h->w_2[l], d_, F_, h->bn_down / (h->pair_down ? 2 : 1));
    }
  }
  if (rc) {
    sfm_destroy(h);
    return rc;
  }
  *out = h;
  return SFM_OK;
}

void sfm_destroy(sfm_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  for (cudaGraphExec_t e : h->graph_exec)
    if (e) cudaGraphExecDestroy(e);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  for (void* p : h->owned) cudaFree(p);
  if (h->h_err) cudaFreeHost((void*)h->h_err);
  delete h;
}

int sfm_session_open(sfm_handle* h, int cache_units, int* session) {
  if (!h || !session || cache_units < 1) return SFM_EINVAL;
  int slot = -1;
  for (int i = 0; i < (int)h->sessions.size(); ++i)
    if (!h->sessions[i].open) {
      slot = i;
      break;
    }
  if (slot < 0) return SFM_ECAPACITY;
  const long long rows = (long long)cache_units * h->cfg.unit_kv_tokens + h->n_tok;
  if (h->pool_used + rows > h->cfg.pool_tokens) return SFM_ECAPACITY;
  Session& s = h->sessions[slot];
  s.open = true;
  s.cache_units = cache_units;
  s.base_row = h->pool_used;
  s.units = 0;
  h->pool_used += rows;
  *session = slot;
  return SFM_OK;
}

int sfm_session_reset(sfm_handle* h, int session) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  h->sessions[session].units = 0;
  return SFM_OK;
}

int sfm_session_get_info(const sfm_handle* h, int session, sfm_session_info* out) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  if (!out) return SFM_EINVAL;
  const Session& s = h->sessions[session];
  out->cache_units = s.cache_units;
  out->units_appended = s.units;
  out->valid_tokens = valid_tokens(h, s);
  out->p0 = s.units * h->cfg.unit_kv_tokens;
  out->base_row = s.base_row;
  return SFM_OK;
}

}  // extern "C"

namespace {

// Appends n_tok / T_u units of a slice whose rows hold src_heads heads; the cache
// takes heads [head0, head0 + H) of each row (all of them when src_heads == H).
int kvcache_append(sfm_handle* h, int session, const void* k, const void* v, int n_tok,
                   int src_heads, int head0, void* stream) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return SFM_EINVAL;
  const int H = h->cfg.n_heads;
  if (src_heads < H || head0 < 0 || head0 + H > src_heads) return SFM_EINVAL;
  const int src_row_bytes = src_heads * h->cfg.head_dim * h->es;
  const int src_off_bytes = head0 * h->cfg.head_dim * h->es;
  if (src_off_bytes % 16 || src_row_bytes % 16) return SFM_EINVAL;
  const int T = h->cfg.unit_kv_tokens;
  if (n_tok <= 0 || n_tok % T) return SFM_EINVAL;
  Session& s = h->sessions[session];
  long long n_units = n_tok / T;
  if (!h->cfg.ring && s.units + n_units > s.cache_units) return SFM_ECAPACITY;
  // With the ring on, only the last cache_units units of a long slice survive.
  long long skip = n_units > s.cache_units ? n_units - s.cache_units : 0;
  const long long first = s.units + skip;
  const size_t row_bytes = (size_t)h->hd * h->es;
  const char* ks = (const char*)k + skip * T * (size_t)src_row_bytes;
  const char* vs = (const char*)v + skip * T * (size_t)src_row_bytes;
  // the kernel reads rows layer * n_tok + t of the caller's slice; with a skip,
  // each layer's rows start skip * T rows later inside that layer
  ProfScope ps(SFM_PROF_APPEND, (cudaStream_t)stream);
  if (skip) {
    // copy layer by layer so the per-layer source stride stays n_tok
    for (int l = 0; l < h->cfg.n_layers; ++l) {
      rc = launch_kv_append(ks + (size_t)l * n_tok * src_row_bytes,
                            vs + (size_t)l * n_tok * src_row_bytes, h->layer_k(l), h->layer_v(l),
                            1, h->cfg.pool_tokens, (int)row_bytes, (int)((n_units - skip) * T), T,
                            s.base_row, first % s.cache_units, s.cache_units, (cudaStream_t)stream,
                            src_row_bytes, src_off_bytes);
      if (rc) return rc;
    }
  } else {
    rc = launch_kv_append(k, v, h->k_pool, h->v_pool, h->cfg.n_layers, h->cfg.pool_tokens,
                          (int)row_bytes, n_tok, T, s.base_row, first % s.cache_units,
                          s.cache_units, (cudaStream_t)stream, src_row_bytes, src_off_bytes);
    if (rc) return rc;
  }
  s.units += n_units;
  return SFM_OK;
}

}  // namespace

extern "C" {

int sfm_kvcache_append(sfm_handle* h, int session, const void* k, const void* v, int n_tok,
                       void* stream) {
  if (!h) return SFM_EINVAL;
  return kvcache_append(h, session, k, v, n_tok, h->cfg.n_heads, 0, stream);
}

int sfm_kvcache_append_heads(sfm_handle* h, int session, const void* k, const void* v, int n_tok,
                             int src_heads, int head0, void* stream) {
  if (!h) return SFM_EINVAL;
  return kvcache_append(h, session, k, v, n_tok, src_heads, head0, stream);
}

int sfm_kvcache_read(const sfm_handle* h, int session, int layer, long long row0,
                     long long n_rows, void* k_dst, void* v_dst, void* stream) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  const Session& s = h->sessions[session];
  const long long cap = (long long)s.cache_units * h->cfg.unit_kv_tokens + h->n_tok;
  if (layer < 0 || layer >= h->cfg.n_layers || row0 < 0 || n_rows < 0 || row0 + n_rows > cap)
    return SFM_EINVAL;
  if (n_rows > 0 && (!k_dst || !v_dst || !aligned16(k_dst) || !aligned16(v_dst)))
    return SFM_EINVAL;
  return launch_kv_read(h->k_pool, h->v_pool, k_dst, v_dst, layer, h->cfg.pool_tokens,
                        h->hd * h->es, s.base_row + row0, n_rows, (cudaStream_t)stream);
}

int sfm_set_graph_mode(sfm_handle* h, int enabled) {
  if (!h || (enabled != 0 && enabled != 1)) return SFM_EINVAL;
  h->graphs = enabled != 0;
  if (!h->graphs)
    for (cudaGraphExec_t& e : h->graph_exec)
      if (e) {
        // launches already enqueued keep their copy of the graph
        cudaGraphExecDestroy(e);
        e = nullptr;
      }
  return SFM_OK;
}

int sfm_denoise_step(sfm_handle* h, int session, float* z, float tau_from, float tau_to,
                     float* v_out, void* stream) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  if (!h->has_weights || !z || !isfinite(tau_from) || !isfinite(tau_to)) return SFM_EINVAL;
  if (v_out == z) return SFM_EINVAL;   // the step writes both
  if ((rc = device_error_pending(h))) return rc;
  const float taus[2] = {tau_from, tau_to};
  float* zs[1] = {z};
  float* vs[1] = {v_out};
  return solve(h, 1, &session, zs, taus, 2, vs, (cudaStream_t)stream);
}

int sfm_fm_solve(sfm_handle* h, int session, float* z, const float* taus, int n_taus,
                 void* stream) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  if (!h->has_weights || !z) return SFM_EINVAL;
  if ((rc = check_taus(taus, n_taus))) return rc;
  if ((rc = device_error_pending(h))) return rc;
  float* zs[1] = {z};
  return solve(h, 1, &session, zs, taus, n_taus, nullptr, (cudaStream_t)stream);
}

int sfm_fm_solve_batched(sfm_handle* h, int n_sessions, const int* sessions, float* const* z,
                         const float* taus, int n_taus, void* stream) {
  if (!h || !sessions || !z || n_sessions < 1) return SFM_EINVAL;
  if (!h->has_weights) return SFM_EINVAL;
  if (n_sessions > h->cfg.max_sessions) return SFM_ECAPACITY;
  int rc;
  // distinct sessions (each writes its unit's K/V into its own scratch rows) and
  // distinct latents (each session's Euler update writes its own z)
  for (int i = 0; i < n_sessions; ++i) {
    if ((rc = session_ok(h, sessions[i]))) return rc;
    if (!z[i]) return SFM_EINVAL;
    for (int j = 0; j < i; ++j)
      if (sessions[j] == sessions[i] || z[j] == z[i]) return SFM_EINVAL;
  }
  if ((rc = check_taus(taus, n_taus))) return rc;
  if ((rc = device_error_pending(h))) return rc;
  return solve(h, n_sessions, sessions, z, taus, n_taus, nullptr, (cudaStream_t)stream);
}

int sfm_fm_solve_guided_batched(sfm_handle* h, int n_pairs, const int* sessions,
                                const int* uncond_sessions, float* const* z, const float* taus,
                                int n_taus, float scale, float* const* v_out, void* stream) {
  if (!h || !sessions || !uncond_sessions || !z || n_pairs < 1) return SFM_EINVAL;
  if (!h->has_weights || !isfinite(scale)) return SFM_EINVAL;
  if (n_pairs > kMaxBatch / 2 || 2 * n_pairs > h->cfg.max_sessions) return SFM_ECAPACITY;
  int rc;
  int ids[kMaxBatch];
  float* zs[kMaxBatch];
  float* vs[kMaxBatch];
  for (int p = 0; p < n_pairs; ++p) {
    if (!z[p]) return SFM_EINVAL;
    // each pair's Euler update writes its own z and velocity
    for (int q = 0; q < n_pairs; ++q) {
      if (q < p && (z[q] == z[p] || (v_out && v_out[p] && v_out[q] == v_out[p]))) return SFM_EINVAL;
      if (v_out && v_out[p] && v_out[p] == z[q]) return SFM_EINVAL;
    }
    ids[2 * p] = sessions[p];
    ids[2 * p + 1] = uncond_sessions[p];
    zs[2 * p] = zs[2 * p + 1] = z[p];
    vs[2 * p] = vs[2 * p + 1] = v_out ? v_out[p] : nullptr;
  }
  // every session (conditional or not) distinct: each evaluation writes its
  // unit's K/V into its own session's scratch rows
  for (int i = 0; i < 2 * n_pairs; ++i) {
    if ((rc = session_ok(h, ids[i]))) return rc;
    for (int j = 0; j < i; ++j)
      if (ids[j] == ids[i]) return SFM_EINVAL;
  }
  if ((rc = check_taus(taus, n_taus))) return rc;
  if ((rc = device_error_pending(h))) return rc;
  Guidance gd;
  gd.on = true;
  gd.scale = scale;
  return solve(h, 2 * n_pairs, ids, zs, taus, n_taus, vs, (cudaStream_t)stream, gd);
}

int sfm_fm_solve_guided(sfm_handle* h, int session, int uncond_session, float* z,
                        const float* taus, int n_taus, float scale, void* stream) {
  return sfm_fm_solve_guided_batched(h, 1, &session, &uncond_session, &z, taus, n_taus, scale,
                                     nullptr, stream);
}

int sfm_velocity_units(sfm_handle* h, int session, int n_units, const float* const* z,
                       const float* taus, float* const* v_out, int commit, void* stream) {
  int rc = session_ok(h, session);
  if (rc) return rc;
  if (!h->has_weights || !z || !taus || !v_out || n_units < 1 || (commit != 0 && commit != 1))
    return SFM_EINVAL;
  if (n_units > h->cfg.max_sessions || n_units > kMaxBatch) return SFM_ECAPACITY;
  for (int u = 0; u < n_units; ++u) {
    if (!z[u] || !v_out[u] || !isfinite(taus[u])) return SFM_EINVAL;
    for (int q = 0; q < n_units; ++q)
      if (v_out[u] == z[q] || (q < u && v_out[q] == v_out[u])) return SFM_EINVAL;
  }
  Session& se = h->sessions[session];
  const long long N = h->n_tok, T = h->cfg.unit_kv_tokens;
  const long long valid = valid_tokens(h, se);
  // the pass's own K/V go to the rows after the valid cache: they must fit the
  // session's region (its slots plus the unit's scratch rows)
  if (valid + n_units * N > (long long)se.cache_units * T + N) return SFM_ECAPACITY;
  if (commit) {
    if (T != N) return SFM_EUNSUPPORTED;              // a committed unit is one cache unit
    if (se.units + n_units > se.cache_units) return SFM_ECAPACITY;   // no ring wrap
  }
  if ((rc = device_error_pending(h))) return rc;
  Pass ps;
  BatchDesc& b = ps.b;
  memset(&b, 0, sizeof(b));
  b.n = n_units;
  b.n_tok = (int)N;
  b.n_video = h->cfg.n_video;
  b.per_tau = 1;
  for (int u = 0; u < n_units; ++u) {
    b.base[u] = se.base_row;
    b.valid[u] = (int)(valid + u * N);           // unit u's K/V rows follow the earlier units'
    b.p0[u] = se.units * T + u * N;
    b.t_unit[u] = se.units + u;
    b.tau[u] = taus[u];
  }
  AttnDesc& a = ps.a;
  memset(&a, 0, sizeof(a));
  a.n = 1;
  a.rows_per = (int)(n_units * N);
  a.unit_rows = (int)N;
  a.kbase[0] = se.base_row;
  a.nkeys[0] = (int)(valid + n_units * N);
  // one step of zero length: the head kernel writes v and leaves z as it is
  const float zero_step[2] = {0.f, 0.f};
  // the latents are only read (a zero-length step writes no z)
  rc = solve_pass(h, ps, const_cast<float* const*>(z), zero_step, 2, v_out, (cudaStream_t)stream,
                  Guidance{}, kGraphUnits);
  if (rc) return rc;
  if (commit) se.units += n_units;               // the rows are the next slots already
  return SFM_OK;
}

// The standalone call chooses its split count for a 148-SM B200 whatever the
// device, so the workspace it needs is a pure function of the shape.
constexpr int kStandaloneSms = 148;

size_t sfm_attention_workspace_bytes(int n_q, int n_kv, int n_heads, int head_dim, int dtype) {
  if (dtype != SFM_DTYPE_BF16 || n_q < 1 || n_kv < 1 || n_heads < 1 || head_dim != 128) return 0;
  const int splits = attention_tc_splits(n_q, 1, n_kv, n_heads, kStandaloneSms);
  return attention_workspace_bytes(n_q, n_heads, splits);
}

}  // extern "C"

namespace {

// Device address of g_call_err in the current context.  The address is kept per
// (device, context): after a cudaDeviceReset the primary context, and with it the
// module holding the variable, is new, so the address is resolved again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
std::mutex g_err_mu;
CtxGetCurrentFn g_ctx_current = nullptr;
struct ErrSlot {
  CUcontext ctx = nullptr;
  int* ptr = nullptr;
};
ErrSlot g_err_slot[64];
int g_call_fault = 0;
unsigned long long g_call_wait_ns = 0;

}  // namespace

namespace sfm {
int current_context(void** ctx) {
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = (CtxGetCurrentFn)fn;
    else
      cudaGetLastError();
  });
  CUcontext c = nullptr;
  if (!g_ctx_current || g_ctx_current(&c) != CUDA_SUCCESS) return SFM_ECUDA;
  *ctx = (void*)c;
  return SFM_OK;
}
}  // namespace sfm

namespace {

int call_guard(Guard* gd) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev < 0 || dev >= 64) return SFM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_err_mu);
  CUcontext ctx = nullptr;
  if (current_context((void**)&ctx)) return SFM_ECUDA;
  ErrSlot& slot = g_err_slot[dev];
  if (!ctx || slot.ctx != ctx || !slot.ptr) {
    // resolving the symbol also makes the runtime bring up the device's context
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_call_err);
    if (e != cudaSuccess || !p) return record_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    if (!ctx && (current_context((void**)&ctx) || !ctx)) return SFM_ECUDA;
    slot.ctx = ctx;
    slot.ptr = (int*)p;
  }
  gd->err = slot.ptr;
  gd->fault = g_call_fault;
  if (g_call_wait_ns) gd->wait_ns = g_call_wait_ns;
  return SFM_OK;
}

// Standalone attention, every key visible (unit_tokens = 0) or block-causal over
// query units of unit_tokens with the first n_kv - n_q keys a shared prefix.
int attention_call(const void* q, const void* k, const void* v, void* o, int n_q, int n_kv,
                   int unit_tokens, int n_heads, int head_dim, int dtype, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || n_q < 1 || n_kv < 1 || n_heads < 1) return SFM_EINVAL;
  if (dtype != SFM_DTYPE_BF16 && dtype != SFM_DTYPE_FP32) return SFM_EINVAL;
  if (dtype == SFM_DTYPE_BF16 && head_dim != 128) return SFM_EUNSUPPORTED;
  if (dtype == SFM_DTYPE_FP32 && (head_dim % 32 || head_dim > 128 || head_dim < 32))
    return SFM_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SFM_EINVAL;
  const size_t need = sfm_attention_workspace_bytes(n_q, n_kv, n_heads, head_dim, dtype);
  if (workspace_bytes < need || (need && (!workspace || !aligned16(workspace)))) return SFM_EINVAL;
  AttnDesc a{};
  a.n = 1;
  a.rows_per = n_q;
  a.unit_rows = unit_tokens;
  a.kbase[0] = 0;
  a.nkeys[0] = n_kv;
  if (dtype == SFM_DTYPE_FP32)
    return launch_attention(a, q, k, v, o, n_heads, head_dim, dtype, 1, nullptr, nullptr, stream);
  // a block-causal call uses at most the splits of the every-key-visible one, so the
  // workspace sfm_attention_workspace_bytes sizes serves both
  int splits = attention_tc_splits(n_q, 1, n_kv, n_heads, kStandaloneSms);
  if (unit_tokens > 0) {
    const int bc = attention_tc_splits(n_q, 1, n_kv, n_heads, kStandaloneSms, unit_tokens);
    splits = bc < splits ? bc : splits;
  }
  float *o_part = nullptr, *lse_part = nullptr;
  if (splits > 1) {
    o_part = (float*)workspace;
    lse_part = o_part + (size_t)splits * n_q * n_heads * 128;
  }
  CUtensorMap mq, mk, mv;
  int rc = make_rows_map(&mq, q, n_q, n_heads, kAttnQBoxRows);
  if (!rc) rc = make_rows_map(&mk, k, n_kv, n_heads, kAttnKVBoxRows);
  if (!rc) rc = make_rows_map(&mv, v, n_kv, n_heads, kAttnKVBoxRows);
  Guard gd;
  if (!rc) rc = call_guard(&gd);
  if (rc) return rc;
  return launch_attention_tc(mq, mk, mv, a, 0, n_heads, splits, o, o_part, lse_part, gd, stream);
}

}  // namespace

extern "C" {

int sfm_attention(const void* q, const void* k, const void* v, void* o, int n_q, int n_kv,
                  int n_heads, int head_dim, int dtype, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return attention_call(q, k, v, o, n_q, n_kv, 0, n_heads, head_dim, dtype, workspace,
                        workspace_bytes, (cudaStream_t)stream);
}

int sfm_attention_block_causal(const void* q, const void* k, const void* v, void* o, int n_q,
                               int n_kv, int unit_tokens, int n_heads, int head_dim, int dtype,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (unit_tokens < 1 || n_kv < n_q) return SFM_EINVAL;
  return attention_call(q, k, v, o, n_q, n_kv, unit_tokens, n_heads, head_dim, dtype, workspace,
                        workspace_bytes, (cudaStream_t)stream);
}

int sfm_fm_solve_exact_velocity(const sfm_handle* h, const float* z0, float* z, const float* taus,
                                int n_taus, void* stream) {
  if (!h || !z0 || !z) return SFM_EINVAL;
  int rc = check_taus(taus, n_taus);
  if (rc) return rc;
  // the velocity (z - z0) / tau is evaluated at every tau but the last
  for (int i = 0; i + 1 < n_taus; ++i)
    if (!(taus[i] > 0.f)) return SFM_EINVAL;
  const long long n = (long long)h->n_tok * h->cfg.c_lat;
  for (int i = 0; i + 1 < n_taus; ++i)
    if ((rc = launch_exact_velocity_euler(z, z0, taus[i], taus[i + 1], n, (cudaStream_t)stream)))
      return rc;
  return SFM_OK;
}

int sfm_euler_update(float* z, const float* v, float dtau, long long n, void* stream) {
  if (n < 0 || (n > 0 && (!z || !v || !aligned16(z) || !aligned16(v))) || !isfinite(dtau))
    return SFM_EINVAL;
  return launch_euler(z, v, dtau, n, (cudaStream_t)stream);
}

int sfm_check_device_error(const sfm_handle* h, int* code) {
  if (!h || !code) return SFM_EINVAL;
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return record_cuda(e);
  *code = v;
  return SFM_OK;
}

int sfm_clear_device_error(sfm_handle* h) {
  if (!h) return SFM_EINVAL;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemset(h->d_err, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return record_cuda(e);
  if (h->h_err) *h->h_err = 0;
  return SFM_OK;
}

int sfm_check_call_error(int* code) {
  if (!code) return SFM_EINVAL;
  Guard gd;
  int rc = call_guard(&gd);
  if (rc) return rc;
  int v = 0;
  const int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, gd.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(gd.err, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return record_cuda(e);
  *code = v;
  return SFM_OK;
}

int sfm_test_fault(sfm_handle* h, int faults, long long wait_ns) {
  if (faults & ~(SFM_FAULT_ATTN_NO_LOADS | SFM_FAULT_GEMM_NO_LOADS)) return SFM_EINVAL;
  if (wait_ns != 0 && (wait_ns < 10000LL || wait_ns > 10000000000LL)) return SFM_EINVAL;
  const unsigned long long ns = wait_ns ? (unsigned long long)wait_ns : sm100::kWaitNs;
  if (h) {
    h->gd.fault = faults;
    h->gd.wait_ns = ns;
  } else {
    std::lock_guard<std::mutex> lock(g_err_mu);
    g_call_fault = faults;
    g_call_wait_ns = wait_ns ? ns : 0;
  }
  return SFM_OK;
}

int sfm_get_plan(const sfm_handle* h, sfm_plan* out) {
  if (!h || !out) return SFM_EINVAL;
  memset(out, 0, sizeof(*out));
  const int bn[4] = {h->bn_qkv, h->bn_o, h->bn_up, h->bn_down};
  const bool pr[4] = {h->pair_qkv, h->pair_o, h->pair_up, h->pair_down};
  const int ks[4] = {1, h->ksplit_o, 1, h->ksplit_down};
  for (int i = 0; i < 4; ++i) {
    out->block_n[i] = bn[i];
    out->pair[i] = pr[i] ? 1 : 0;
    out->k_splits[i] = ks[i];
  }
  out->fused_norm = h->has_weights && h->cfg.dtype == SFM_DTYPE_BF16 ? 1 : 0;
  return SFM_OK;
}

int sfm_attention_batch_splits(int n_sessions, int rows_per_session, const long long* n_keys,
                               int n_heads, int sms, int* splits) {
  if (!n_keys || !splits || n_sessions < 1 || n_sessions > kMaxBatch || rows_per_session < 1 ||
      n_heads < 1 || sms < 1)
    return SFM_EINVAL;
  AttnDesc a{};
  a.n = n_sessions;
  a.rows_per = rows_per_session;
  for (int i = 0; i < n_sessions; ++i) {
    if (n_keys[i] < 1 || n_keys[i] > INT_MAX) return SFM_EINVAL;
    a.nkeys[i] = (int)n_keys[i];
  }
  attention_tc_splits_batch(a, n_heads, sms, splits);
  return SFM_OK;
}

int sfm_linear(const void* x, const void* w, void* y, int M, int N, int K, int epilogue,
               int dtype, void* stream) {
  if (!x || !w || !y || M < 1 || N < 1 || K < 1) return SFM_EINVAL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return SFM_EINVAL;
  int epi;
  switch (epilogue) {
    case SFM_LINEAR_F32: epi = EPI_F32; break;
    case SFM_LINEAR_OUT: epi = EPI_STORE; break;
    case SFM_LINEAR_GELU: epi = EPI_GELU; break;
    case SFM_LINEAR_RESID: epi = EPI_RESID; break;
    default: return SFM_EINVAL;
  }
  if (dtype == SFM_DTYPE_FP32) {
    if (N % 64 || K % 16) return SFM_EUNSUPPORTED;
    return launch_gemm(x, w, y, M, N, K, epi, dtype, (cudaStream_t)stream);
  }
  if (dtype != SFM_DTYPE_BF16) return SFM_EINVAL;
  if (N % 128 || K % 64) return SFM_EUNSUPPORTED;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool pair = gemm_tc_pair(M, N, 0, epi, sms);
  const int bn = gemm_tc_block_n(M, N, 0, epi, sms, pair);
  if (!bn) return SFM_EUNSUPPORTED;
  CUtensorMap ma, mb;
  int rc = make_a_map(&ma, x, M, K);
  if (!rc) rc = make_b_map(&mb, w, N, K, pair ? bn / 2 : bn);
  Guard gd;
  if (!rc) rc = call_guard(&gd);
  if (rc) return rc;
  return launch_gemm_tc(ma, mb, gemm_args(M, N, K, epi, y, N, gd, bn, pair), sms,
                        (cudaStream_t)stream);
}

const char* sfm_strerror(int status) {
  switch (status) {
    case SFM_OK: return "ok";
    case SFM_EINVAL: return "invalid argument";
    case SFM_ECAPACITY: return "capacity exceeded";
    case SFM_ESESSION: return "unknown or closed session";
    case SFM_ECUDA: return "CUDA error";
    case SFM_ENOMEM: return "device allocation failed";
    case SFM_EUNSUPPORTED: return "unsupported shape";
    case SFM_EDEVICE: return "a kernel gave up a bounded wait (clear with sfm_clear_device_error)";
    default: return "unknown status";
  }
}

int sfm_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
