// a2. Top-k with one CTA per request (the DSA top-k subset, "Related papers: SparseServe"
// page, DSA abstract; ties to the lower position, output in ascending position order).
//
// The whole request is handled by one 1,024-thread CTA reading its scores from L2, so a
// small batch occupies few SMs (the attention that follows can start its prologue on the
// others) and no cluster barrier or distributed-shared-memory round is needed.  Scores are
// compared as order-preserving u32 keys.  Warp w owns a contiguous segment of the request.
//
//   pass A   every warp counts the top 11 bits of its keys into its own 2,048-bin
//            histogram (two 16-bit counts per word, so 32 of them fit in 128 KB); the
//            merged histogram gives bin t0 holding the k-th largest key.
//   pass B   every warp walks its segment in position order and lists the keys at or
//            above bin t0 (offset and key): every output is on these lists.
//   select   two radix passes (11 + 10 bits) over the listed keys of bin t0 give the
//            exact k-th key T and how many keys equal to T are taken.
//   emit     per-warp counts, a block scan, and each warp writes its taken keys in order.
// A list that would overflow sends the CTA to a slower exact path: two more radix passes
// and the emit straight from the scores.
#pragma once
#include "common.cuh"
#include "topk.cuh"

namespace ls {

constexpr int kRowThreads = 1024;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowList = 512;                       // list entries per warp
constexpr int kRowHistWords = 1024;                 // 2,048 bins, two 16-bit counts per word
constexpr int kRowSmem = kRowWarps * kRowHistWords * 4;  // 128 KB: histograms, then the lists
static_assert(kRowWarps * kRowList * 6 <= kRowSmem, "lists fit where the histograms were");
constexpr int kRowMaxKeys = kRowWarps * 65532;      // 16-bit per-warp offsets and counts

// Bin of the k_rem-th largest key among the counts hist[0 .. nbins) (bins scanned from the
// top): every thread returns the same (bin, keys in higher bins).
__device__ __forceinline__ void row_find_bin(const uint32_t* hist, int nbins, uint32_t k_rem,
                                             unsigned long long* scan_tmp, int* s_bin, uint32_t* s_above) {
  const int tid = threadIdx.x;
  const int per = nbins / kRowThreads;  // 2 or 1
  uint32_t mine = 0;
  for (int j = 0; j < per; ++j) mine += hist[nbins - 1 - (tid * per + j)];
  unsigned long long tot;
  uint32_t above = (uint32_t)block_excl_scan_u64(mine, scan_tmp, &tot);
  for (int j = 0; j < per; ++j) {
    const int d = nbins - 1 - (tid * per + j);
    const uint32_t h = hist[d];
    if (above < k_rem && above + h >= k_rem) {
      *s_bin = d;
      *s_above = above;
    }
    above += h;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kRowThreads, 1) topk_row(const TopkParams p) {
  extern __shared__ __align__(16) uint32_t row_smem[];
  __shared__ uint32_t hist[2048];
  __shared__ unsigned long long scan_tmp[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_ovf;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const uint32_t lt = (1u << lane) - 1u;
  const int k = p.k;
  griddep_wait();  // the scores come from the kernel before
  if (p.clear && threadIdx.x == 0) p.clear[blockIdx.x] = 0;
  griddep_launch_dependents();

  const long long nll = ((long long)p.lens[b] * p.len_mul + p.len_div - 1) / p.len_div;
  const bool bad = nll < 0 || nll > p.len_limit || nll > kRowMaxKeys;
  const int n = bad ? 0 : (int)nll;
  if (bad && tid == 0) flag(LS_DEV_BOUNDS);
  const float* row = p.scores + (size_t)b * p.stride;
  if (n < k) {
    // fewer candidates than k: all of them, in order, then -1 padding
    for (int i = tid; i < k; i += kRowThreads) {
      if (p.idx) p.idx[(size_t)b * k + i] = i < n ? topk_pos(p, b, i) : -1;
      if (p.sel) p.sel[(size_t)b * k + i] = i < n ? row[i] : 0.f;
    }
    if (p.thr && tid == 0) p.thr[b] = -INFINITY;
    if (p.done) {
      __syncthreads();
      count_done(p.done + b);
    }
    return;
  }
  const int seg = ((n + kRowWarps * 4 - 1) / (kRowWarps * 4)) * 4;  // keys per warp, multiple of 4
  const int i0 = min(n, warp * seg), i1 = min(n, i0 + seg);

  // ---- pass A: per-warp histograms of the top 11 bits
  for (int w = tid; w < kRowWarps * kRowHistWords; w += kRowThreads) row_smem[w] = 0;
  if (tid == 0) s_ovf = 0;
  __syncthreads();
  {
    uint32_t* wh = row_smem + warp * kRowHistWords;
    auto count4 = [&](float4 v, int i) {
      const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i + e < i1) {
          const uint32_t bin = float_key(f[e]) >> 21;
          atomicAdd(&wh[bin >> 1], 1u << ((bin & 1u) << 4));
        }
    };
    // four 512-byte rows of the segment in flight per warp
    for (int base = i0; base < i1; base += 4 * 128) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 128 + lane * 4;
        if (i + 3 < i1) {
          v[u] = *(const float4*)(row + i);
        } else {
          v[u] = make_float4(i < i1 ? row[i] : 0.f, i + 1 < i1 ? row[i + 1] : 0.f, i + 2 < i1 ? row[i + 2] : 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) count4(v[u], base + u * 128 + lane * 4);
    }
  }
  __syncthreads();
  {
    uint32_t c0 = 0, c1 = 0;  // word tid = bins 2*tid and 2*tid + 1
    for (int w = 0; w < kRowWarps; ++w) {
      const uint32_t v = row_smem[w * kRowHistWords + tid];
      c0 += v & 0xFFFFu;
      c1 += v >> 16;
    }
    hist[2 * tid] = c0;
    hist[2 * tid + 1] = c1;
  }
  __syncthreads();
  row_find_bin(hist, 2048, (uint32_t)k, scan_tmp, &s_bin, &s_above);
  const uint32_t t0 = (uint32_t)s_bin;
  uint32_t k_rem = (uint32_t)k - s_above;  // keys of bin t0 still to take (>= 1)
  __syncthreads();                         // the histograms are read; their space becomes the lists

  // ---- pass B: each warp's ordered list of its keys at or above bin t0
  uint16_t* loff = (uint16_t*)row_smem + warp * kRowList;
  uint32_t* lkey = row_smem + kRowWarps * kRowList / 2 + warp * kRowList;
  uint32_t nl = 0;
  for (int base = i0; base < i1; base += 4 * 32) {
    uint32_t key[4];
    bool sel[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * 32 + lane;
      key[u] = i < i1 ? float_key(row[i]) : 0u;
      sel[u] = i < i1 && (key[u] >> 21) >= t0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t m = __ballot_sync(0xffffffffu, sel[u]);
      if (sel[u]) {
        const uint32_t o = nl + __popc(m & lt);
        if (o < (uint32_t)kRowList) {
          loff[o] = (uint16_t)(base + u * 32 + lane - i0);
          lkey[o] = key[u];
        }
      }
      nl += __popc(m);
    }
  }
  if (lane == 0 && nl > (uint32_t)kRowList) s_ovf = 1;
  __syncthreads();

  uint32_t T, R;
  if (!s_ovf) {
    // ---- exact k-th key among the listed keys of bin t0: bits 20..10, then 9..0
    uint32_t prefix = t0;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0, nb = pass == 0 ? 2048 : 1024, hs = pass == 0 ? 21 : 10;
      for (int d = tid; d < 2048; d += kRowThreads) hist[d] = 0;
      __syncthreads();
      for (uint32_t j = lane; j < nl; j += 32) {
        const uint32_t key = lkey[j];
        if ((key >> hs) == prefix) atomicAdd(&hist[(key >> shift) & (uint32_t)(nb - 1)], 1u);
      }
      __syncthreads();
      row_find_bin(hist, nb, k_rem, scan_tmp, &s_bin, &s_above);
      prefix = (prefix << (pass == 0 ? 11 : 10)) | (uint32_t)s_bin;
      k_rem -= s_above;
      __syncthreads();
    }
    T = prefix;
    R = k_rem;  // keys equal to T to take, lowest positions first
    // ---- per-warp counts over the list, their block scan, then the ordered emit
    uint32_t g = 0, e = 0;
    for (uint32_t j = lane; j < nl; j += 32) {
      g += lkey[j] > T ? 1u : 0u;
      e += lkey[j] == T ? 1u : 0u;
    }
    g = __reduce_add_sync(0xffffffffu, g);
    e = __reduce_add_sync(0xffffffffu, e);
    unsigned long long tot;
    const unsigned long long pre_t =
        block_excl_scan_u64(lane == 0 ? (((unsigned long long)g << 32) | e) : 0ull, scan_tmp, &tot);
    const unsigned long long pre = __shfl_sync(0xffffffffu, pre_t, 0);
    const uint32_t gt_pre = (uint32_t)(pre >> 32), eq_pre = (uint32_t)pre;
    uint32_t eq_seen = eq_pre;
    uint32_t out = gt_pre + min(eq_pre, R);
    for (uint32_t jb = 0; jb < nl; jb += 32) {
      const uint32_t j = jb + lane;
      const bool in = j < nl;
      const uint32_t key = in ? lkey[j] : 0u;
      const uint32_t eq_mask = __ballot_sync(0xffffffffu, in && key == T);
      const bool take = in && (key > T || (key == T && eq_seen + __popc(eq_mask & lt) < R));
      const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
      if (take) {
        const uint32_t o = out + __popc(take_mask & lt);
        if (o < (uint32_t)k) {
          const int gi = i0 + loff[j];
          if (p.idx) p.idx[(size_t)b * k + o] = topk_pos(p, b, gi);
          if (p.sel) p.sel[(size_t)b * k + o] = key_float(key);
        }
      }
      out += __popc(take_mask);
      eq_seen += __popc(eq_mask);
    }
  } else {
    // ---- a list overflowed (keys bunched by position): finish from the scores
    uint32_t prefix = t0;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0, nb = pass == 0 ? 2048 : 1024, hs = pass == 0 ? 21 : 10;
      for (int d = tid; d < 2048; d += kRowThreads) hist[d] = 0;
      __syncthreads();
      for (int i = i0 + lane; i < i1; i += 32) {
        const uint32_t key = float_key(row[i]);
        if ((key >> hs) == prefix) atomicAdd(&hist[(key >> shift) & (uint32_t)(nb - 1)], 1u);
      }
      __syncthreads();
      row_find_bin(hist, nb, k_rem, scan_tmp, &s_bin, &s_above);
      prefix = (prefix << (pass == 0 ? 11 : 10)) | (uint32_t)s_bin;
      k_rem -= s_above;
      __syncthreads();
    }
    T = prefix;
    R = k_rem;
    uint32_t g = 0, e = 0;
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < i1 ? float_key(row[i]) : 0u;
      g += __popc(__ballot_sync(0xffffffffu, i < i1 && key > T));
      e += __popc(__ballot_sync(0xffffffffu, i < i1 && key == T));
    }
    unsigned long long tot;
    const unsigned long long pre_t =
        block_excl_scan_u64(lane == 0 ? (((unsigned long long)g << 32) | e) : 0ull, scan_tmp, &tot);
    const unsigned long long pre = __shfl_sync(0xffffffffu, pre_t, 0);
    const uint32_t gt_pre = (uint32_t)(pre >> 32), eq_pre = (uint32_t)pre;
    uint32_t eq_seen = eq_pre;
    uint32_t out = gt_pre + min(eq_pre, R);
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      const bool in = i < i1;
      const uint32_t key = in ? float_key(row[i]) : 0u;
      const uint32_t eq_mask = __ballot_sync(0xffffffffu, in && key == T);
      const bool take = in && (key > T || (key == T && eq_seen + __popc(eq_mask & lt) < R));
      const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
      if (take) {
        const uint32_t o = out + __popc(take_mask & lt);
        if (o < (uint32_t)k) {
          if (p.idx) p.idx[(size_t)b * k + o] = topk_pos(p, b, i);
          if (p.sel) p.sel[(size_t)b * k + o] = key_float(key);
        }
      }
      out += __popc(take_mask);
      eq_seen += __popc(eq_mask);
    }
  }
  if (p.thr && tid == 0) p.thr[b] = key_float(T);
  if (p.done) {
    __syncthreads();
    count_done(p.done + b);
  }
}

}  // namespace ls
