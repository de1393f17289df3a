// Attention launch interface shared by the C-ABI and the attention kernels.
#pragma once
#include "common.cuh"

namespace sfm {

constexpr int kMaxSplits = 8;

// Query rows [s * rows_per, (s + 1) * rows_per) of session s attend to key
// rows [kbase[s], kbase[s] + nkeys[s]) of the layer's K/V arrays.
struct AttnDesc {
  int n;
  int rows_per;
  long long kbase[kMaxBatch];
  int nkeys[kMaxBatch];
};

int attention_splits(int rows_per_session, int n_sessions, long long max_keys, int n_heads);
size_t attention_workspace_bytes(long long rows, int n_heads, int n_splits);
int launch_attention(const AttnDesc& a, const void* q, const void* k, const void* v, void* o,
                     int n_heads, int head_dim, int dtype, int n_splits, float* o_part,
                     float* lse_part, cudaStream_t s);

}  // namespace sfm
