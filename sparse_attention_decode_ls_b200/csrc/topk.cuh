// a2. Per-request top-k (the DSA top-k subset of the cached entries; 2,048 per step
// in XM-Sparse's hot-buffer analysis).
//
// One thread-block cluster per request.  Each CTA owns a contiguous slice of the
// request's scores, converts them once to order-preserving 32-bit keys and keeps them
// in shared memory.  Three radix passes (11, 11, 10 bits) build shared-memory
// histograms of the candidates, merged across the cluster through distributed
// shared memory, until the exact k-th key T is known.  The emit pass then writes, in
// ascending position order, every position with key > T plus the lowest-positioned
// ones with key == T -- the tie rule "lower position first".
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace ls {
namespace cg = cooperative_groups;

struct TopkParams {
  int B, k, stride;          // scores row stride (elements, multiple of 4)
  const float* scores;
  const int* lens;           // [B]
  int len_mul, len_div;      // candidate count = ceil(lens[b] * len_mul / len_div)
  int len_limit;             // candidate counts above this are out of range
  const int* unit_list;      // optional: position of candidate i = unit_list[b][i/64]*64 + i%64
  int list_stride;
  int* idx;                  // [B,k] (may be NULL: threshold only)
  float* sel;                // [B,k] (may be NULL)
  float* thr;                // [B] optional: k-th largest score, -inf if fewer than k candidates
  int cache_keys;            // keys of dynamic shared memory available per CTA
};

constexpr int kTopkThreads = 512;
constexpr int kTopkCacheKeys = 40960;  // at most 160 KB of cached keys per CTA

__device__ __forceinline__ int topk_pos(const TopkParams& p, int b, int i) {
  if (!p.unit_list) return i;
  return p.unit_list[(size_t)b * p.list_stride + (i >> 6)] * 64 + (i & 63);
}

template <int CL>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_cluster(const TopkParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t sm_keys[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t red[2048 / CL];
  __shared__ uint32_t ghist[2048];
  __shared__ unsigned long long scan_tmp[32];
  __shared__ unsigned long long cnt_pub;  // this CTA's (n_gt << 32 | n_eq), read by the cluster
  __shared__ int s_found_bin;
  __shared__ uint32_t s_found_above;

  const int b = blockIdx.x / CL;
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int k = p.k;

  long long nll = ((long long)p.lens[b] * p.len_mul + p.len_div - 1) / p.len_div;
  bool bad = nll < 0 || nll > p.len_limit;
  const int n = bad ? 0 : (int)nll;
  if (bad && rank == 0 && tid == 0) flag(LS_DEV_BOUNDS);
  const int Lc = (((n + CL - 1) / CL) + 3) & ~3;
  const int c0 = min(n, rank * Lc);
  const int c1 = min(n, c0 + Lc);
  const int m = c1 - c0;
  const bool cached = Lc <= p.cache_keys;
  const float* row = p.scores + (size_t)b * p.stride;

  auto key_at = [&](int i) -> uint32_t {  // i relative to c0
    return cached ? sm_keys[i] : float_key(row[c0 + i]);
  };

  if (n < k) {
    // fewer candidates than k: all of them, in order, then -1 padding
    for (int i = tid; i < m; i += kTopkThreads) {
      const int gi = c0 + i;
      if (p.idx) p.idx[(size_t)b * k + gi] = topk_pos(p, b, gi);
      if (p.sel) p.sel[(size_t)b * k + gi] = row[gi];
    }
    if (rank == 0) {
      for (int i = n + tid; i < k; i += kTopkThreads) {
        if (p.idx) p.idx[(size_t)b * k + i] = -1;
        if (p.sel) p.sel[(size_t)b * k + i] = 0.f;
      }
      if (p.thr && tid == 0) p.thr[b] = -INFINITY;
    }
    return;  // no distributed shared memory was touched
  }

  if (cached) {
    const int m4 = m & ~3;
    for (int i = tid * 4; i < m4; i += kTopkThreads * 4) {
      const float4 v = *(const float4*)(row + c0 + i);
      sm_keys[i] = float_key(v.x);
      sm_keys[i + 1] = float_key(v.y);
      sm_keys[i + 2] = float_key(v.z);
      sm_keys[i + 3] = float_key(v.w);
    }
    for (int i = m4 + tid; i < m; i += kTopkThreads) sm_keys[i] = float_key(row[c0 + i]);
  }

  uint32_t prefix = 0;
  uint32_t k_rem = (uint32_t)k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass], width = widths[pass];
    const int nbins = 1 << width;
    const uint32_t dmask = (uint32_t)nbins - 1u;
    const int hi_shift = shift + width;  // bits above this pass's digit must equal prefix
    for (int d = tid; d < 2048; d += kTopkThreads) hist[d] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += kTopkThreads) {
      const uint32_t key = key_at(i);
      const bool cand = (hi_shift >= 32) || ((key >> hi_shift) == prefix);
      if (cand) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    cluster.sync();
    // reduce my slice of bins over the cluster
    const int slice = 2048 / CL;
    for (int d = tid; d < slice; d += kTopkThreads) {
      const int gd = rank * slice + d;
      uint32_t s = 0;
      if (gd < nbins) {
#pragma unroll
        for (int c = 0; c < CL; ++c) s += cluster.map_shared_rank(hist, c)[gd];
      }
      red[d] = s;
    }
    cluster.sync();
    for (int d = tid; d < nbins; d += kTopkThreads) ghist[d] = cluster.map_shared_rank(red, d / slice)[d % slice];
    __syncthreads();
    // find the bin holding the k_rem-th largest candidate (bins scanned high to low)
    const int per = nbins / kTopkThreads;  // 4 or 2 bins per thread
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j) mine += ghist[nbins - 1 - (tid * per + j)];
    unsigned long long tot;
    uint32_t above = (uint32_t)block_excl_scan_u64(mine, scan_tmp, &tot);
    for (int j = 0; j < per; ++j) {
      const int d = nbins - 1 - (tid * per + j);
      const uint32_t h = ghist[d];
      if (above < k_rem && above + h >= k_rem) {
        s_found_bin = d;
        s_found_above = above;
      }
      above += h;
    }
    __syncthreads();
    prefix = (prefix << width) | (uint32_t)s_found_bin;
    k_rem -= s_found_above;
    __syncthreads();
  }
  const uint32_t T = prefix;   // exact k-th largest key
  const uint32_t R = k_rem;    // how many keys == T are taken (lowest positions first)

  // ---- emit: each warp owns a contiguous segment (position order) and walks it 32 keys
  // at a time, so shared-memory reads are conflict-free and ballots give the ranks
  const int lane = lane_id(), warp = warp_id();
  constexpr int kWarps = kTopkThreads / 32;
  const int seg = ((m + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int i0 = min(m, warp * seg), i1 = min(m, i0 + seg);
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < i1 ? key_at(i) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < i1 && key > T));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < i1 && key == T));
  }
  // warp totals -> exclusive prefix over warps (block scan on one value per thread)
  const unsigned long long mine = lane == 0 ? (((unsigned long long)n_gt << 32) | n_eq) : 0ull;
  unsigned long long tot;
  const unsigned long long pre_t = block_excl_scan_u64(mine, scan_tmp, &tot);
  const unsigned long long pre = __shfl_sync(0xffffffffu, pre_t, 0);
  if (tid == 0) cnt_pub = tot;
  __syncthreads();
  cluster.sync();
  uint32_t eq_before = 0, out_before = 0;
  for (int c = 0; c < rank; ++c) {
    const unsigned long long v = *cluster.map_shared_rank(&cnt_pub, c);
    const uint32_t g = (uint32_t)(v >> 32), e = (uint32_t)v;
    const uint32_t take = R > eq_before ? min(e, R - eq_before) : 0u;
    out_before += g + take;
    eq_before += e;
  }
  const uint32_t eq_left = R > eq_before ? R - eq_before : 0u;  // ties this CTA may still take
  const uint32_t gt_pre = (uint32_t)(pre >> 32), eq_pre = (uint32_t)pre;
  uint32_t eq_seen = eq_pre;  // keys == T before this lane's current key, CTA-wide
  uint32_t out = out_before + gt_pre + min(eq_pre, eq_left);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    const bool in = i < i1;
    const uint32_t key = in ? key_at(i) : 0u;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, in && key == T);
    const bool take = in && (key > T || (key == T && eq_seen + __popc(eq_mask & lt_mask) < eq_left));
    const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const uint32_t o = out + __popc(take_mask & lt_mask);
      if (o < (uint32_t)k) {
        const int gi = c0 + i;
        if (p.idx) p.idx[(size_t)b * k + o] = topk_pos(p, b, gi);
        if (p.sel) p.sel[(size_t)b * k + o] = key_float(key);
      }
    }
    out += __popc(take_mask);
    eq_seen += __popc(eq_mask);
  }
  if (p.thr && rank == 0 && tid == 0) p.thr[b] = key_float(T);
  cluster.sync();  // keep this CTA's shared memory alive until the cluster is done with it
}

}  // namespace ls
