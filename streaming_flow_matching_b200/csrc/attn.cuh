// Attention launch interface shared by the C-ABI and the attention kernels.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace sfm {

constexpr int kMaxSplits = 16;
// TMA box heights of the tcgen05 attention kernel: query and key / value tiles
// of 128 rows (one 64-dim half of a head per box).
constexpr int kAttnQBoxRows = 128;
constexpr int kAttnKVBoxRows = 128;

// Query rows [s * rows_per, (s + 1) * rows_per) of session s attend to key
// rows [kbase[s], kbase[s] + nkeys[s]) of the layer's K/V arrays.
// unit_rows = 0: every key is visible to every query (the performer form).
// unit_rows = U > 0: block-causal over units of U queries -- the last rows_per
// keys belong to the queries themselves, the keys before them are a prefix
// every query sees, and query i (of its session) sees the prefix plus the keys
// of units <= i / U:  keys [0, attn_key_limit(...)).
struct AttnDesc {
  int n;
  int rows_per;
  int unit_rows;
  long long kbase[kMaxBatch];
  int nkeys[kMaxBatch];
};

__host__ __device__ __forceinline__ int attn_key_limit(int nkeys, int rows_per, int unit_rows,
                                                       int i) {
  if (unit_rows <= 0) return nkeys;
  const int own = (i / unit_rows + 1) * unit_rows;
  return nkeys - rows_per + (own < rows_per ? own : rows_per);
}

size_t attention_workspace_bytes(long long rows, int n_heads, int n_splits);
int launch_attention(const AttnDesc& a, const void* q, const void* k, const void* v, void* o,
                     int n_heads, int head_dim, int dtype, int n_splits, float* o_part,
                     float* lse_part, cudaStream_t s);

// The sessions one merge launch combines, all of the same split count: session
// sess[k] (k < n) owns rows [sess[k] * rows_per, (sess[k] + 1) * rows_per).
struct MergeDesc {
  int rows_per;
  int n;
  int sess[kMaxBatch];
};
int launch_attention_merge(const float* o_part, const float* lse_part, void* o,
                           long long total_rows, int n_heads, int n_splits, const MergeDesc& md,
                           cudaStream_t s);

// tcgen05 attention (bf16, D = 128).  Split count for a batch; the SM count is an input so the choice is
// reproducible (the standalone call assumes 148).
// unit_rows > 0: block-causal (see AttnDesc), which shortens the early query blocks.
int attention_tc_splits(int rows_per_session, int n_sessions, long long max_keys, int n_heads,
                        int sms, int unit_rows = 0);
// A batch whose sessions have their own key counts (AttnDesc::nkeys): one split
// count per session into ns[0 .. a.n); returns the largest.
int attention_tc_splits_batch(const AttnDesc& a, int n_heads, int sms, int* ns);
// mq: map over the query rows [rows][H][128]; mk, mv: maps over the key rows, of
// which this call uses rows kv_row0 + kbase[s] + [0, nkeys[s]).
// gd: error word, wait bound and test-only fault of the launch.
// ns: the split count of each session (1..kMaxSplits); sessions of more than one
// split write fp32 partials to o_part / lse_part ([split][rows][H][D], [split][rows][H])
// that a merge then combines into o.
int launch_attention_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const AttnDesc& a, int kv_row0, int n_heads, const int* ns, void* o,
                        float* o_part, float* lse_part, const Guard& gd, cudaStream_t s);
// every session split n_splits ways
int launch_attention_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const AttnDesc& a, int kv_row0, int n_heads, int n_splits, void* o,
                        float* o_part, float* lse_part, const Guard& gd, cudaStream_t s);

}  // namespace sfm
