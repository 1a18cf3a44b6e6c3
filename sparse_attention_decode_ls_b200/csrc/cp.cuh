// Context-parallel split of one request across GPUs: each GPU scores and selects over its
// own contiguous shard of the context; the shards' (score, position) candidates are
// gathered; every GPU takes the same global top-k of them, attends to the selected rows
// that lie in its shard, and the partial outputs are merged by their log-sum-exp.
//
//   cp_compact_kernel    the gathered candidates of each request, shard after shard, valid
//                        entries only: ascending global positions, ready for the top-k.
//   cp_local_sel_kernel  the global selection restricted to this GPU's shard, as local
//                        positions (-1 elsewhere).
#pragma once
#include "common.cuh"

namespace ls {

struct CpCompactParams {
  int G, B, k, stride;     // stride: row stride of the compacted arrays (>= G*k, % 4 == 0)
  const float* cand_score;  // [G,B,k]
  const int* cand_pos;      // [G,B,k] global positions, -1 after each shard's valid ones
  float* score;             // [B,stride] out
  int* pos;                 // [B,stride] out
  int* count;               // [B] out
};

// One CTA per request, 256 threads: shard g's valid entries land after those of shards < g.
__global__ void __launch_bounds__(256) cp_compact_kernel(const CpCompactParams p) {
  __shared__ int s_off;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) s_off = 0;
  __syncthreads();
  for (int g = 0; g < p.G; ++g) {
    const size_t base = ((size_t)g * p.B + b) * p.k;
    // valid entries come first in each shard's list: count them, 256 at a time
    int n = 0;
    for (int j0 = 0; j0 < p.k; j0 += 256) {
      const int j = j0 + threadIdx.x;
      n += __syncthreads_count(j < p.k && p.cand_pos[base + j] >= 0);
    }
    const int off = s_off;
    for (int j = threadIdx.x; j < n; j += 256) {
      p.score[(size_t)b * p.stride + off + j] = p.cand_score[base + j];
      p.pos[(size_t)b * p.stride + off + j] = p.cand_pos[base + j];
    }
    __syncthreads();
    if (threadIdx.x == 0) s_off = off + n;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.count[b] = s_off;
}

// grid (ceil(k/256), B)
__global__ void __launch_bounds__(256) cp_local_sel_kernel(int B, int k, const int* idx, const int* begin,
                                                           const int* end, int* local) {
  const int b = blockIdx.y, j = blockIdx.x * 256 + threadIdx.x;
  if (j >= k) return;
  const int pos = idx[(size_t)b * k + j], lo = begin[b], hi = end[b];
  local[(size_t)b * k + j] = (pos >= lo && pos < hi) ? pos - lo : -1;
}

}  // namespace ls
