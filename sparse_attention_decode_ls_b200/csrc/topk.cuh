// a2. Per-request top-k (the DSA top-k subset of the cached entries; 2,048 per step
// in XM-Sparse's hot-buffer analysis).
//
// One thread-block cluster per request.  Each CTA owns a contiguous slice of the
// request's scores, converts them once to order-preserving 32-bit keys and keeps them
// in shared memory.  The first radix pass (the top 11 bits) is merged across the
// cluster through distributed shared memory; every CTA then gathers the keys of the bin
// holding the k-th largest key and finishes the exact k-th key T with two local passes
// (11, 10 bits), or, when that bin is too crowded, two more cluster-wide passes.  The
// emit pass then writes, in ascending position order, every position with key > T plus
// the lowest-positioned ones with key == T -- the tie rule "lower position first".
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
  const int* pos_list;       // optional: position of candidate i = pos_list[b * pos_stride + i]
  int pos_stride;
  const int* pos_offset;     // optional [B]: added to every emitted position
  int* idx;                  // [B,k] (may be NULL: threshold only)
  float* sel;                // [B,k] (may be NULL)
  float* thr;                // [B] optional: k-th largest score, -inf if fewer than k candidates
  int cache_keys;            // keys of dynamic shared memory available per CTA
  int* clear;                // optional [B]: set to 0 (a per-request count the next kernel of
                             //   the step adds up; see AttnParams::done)
  int* done;                 // optional [B], zero at launch: every CTA adds 1 once its outputs
                             //   are stored (see AttnParams::ready)
};

constexpr int kTopkThreads = 512;
constexpr int kTopkCacheKeys = 36864;  // at most 144 KB of cached keys per CTA

__device__ __forceinline__ int topk_pos(const TopkParams& p, int b, int i) {
  int pos = i;
  if (p.pos_list) {
    pos = p.pos_list[(size_t)b * p.pos_stride + i];
  } else if (p.unit_list) {
    pos = p.unit_list[(size_t)b * p.list_stride + (i >> 6)] * 64 + (i & 63);
  }
  return p.pos_offset ? pos + p.pos_offset[b] : pos;
}

// Buffers of the fast path (dynamic shared memory after the key cache).
constexpr int kCandCap = 2048;    // per CTA: keys of the threshold bin
constexpr int kCandTotal = 8192;  // all candidates of a request, gathered by CTA 0
constexpr int kWarpList = 512;    // per warp: its keys at or above the threshold bin, in order
constexpr int kTopkExtraBytes = kCandCap * 4 + kCandTotal * 4 + (kTopkThreads / 32) * kWarpList * 2;


// Warp 0: lane c holds CTA c's count of keys above the threshold key (g) and equal to
// it (e).  Ties are taken by lower position, i.e. by lower CTA first, R in all.  The lane
// of this CTA's rank stores how many outputs and how many ties precede the CTA.
#define cluster_prefix(g_, e_, R_, rank_, lane_)                                        \
  do {                                                                                  \
    uint32_t _e_incl = (e_);                                                            \
    _Pragma("unroll") for (int _o = 1; _o < 32; _o <<= 1) {                             \
      const uint32_t _y = __shfl_up_sync(0xffffffffu, _e_incl, _o);                     \
      if ((lane_) >= _o) _e_incl += _y;                                                 \
    }                                                                                   \
    const uint32_t _eqb = _e_incl - (e_);                                               \
    const uint32_t _take = (R_) > _eqb ? min((e_), (R_) - _eqb) : 0u;                   \
    uint32_t _o_incl = (g_) + _take;                                                    \
    _Pragma("unroll") for (int _o = 1; _o < 32; _o <<= 1) {                             \
      const uint32_t _y = __shfl_up_sync(0xffffffffu, _o_incl, _o);                     \
      if ((lane_) >= _o) _o_incl += _y;                                                 \
    }                                                                                   \
    if ((lane_) == (rank_)) {                                                           \
      s_out_before = _o_incl - ((g_) + _take);                                          \
      s_eq_before = _eqb;                                                               \
    }                                                                                   \
  } while (0)

template <int CL>
// At most 64 registers: two CTAs per SM, so that all clusters of a batch are resident at once.
__global__ void __launch_bounds__(kTopkThreads, 2) topk_cluster(const TopkParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t sm_keys[];  // [cache_keys] then candidate buffers
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t red[2048 / CL];
  __shared__ uint32_t ghist[2048];
  __shared__ unsigned long long scan_tmp[32];
  __shared__ unsigned long long cnt_pub;  // fallback path: this CTA's (n_gt << 32 | n_eq)
  __shared__ int s_found_bin;
  __shared__ uint32_t s_found_above;
  // fast path
  __shared__ uint32_t s_ncand, s_nabove, s_overflow;
  __shared__ uint32_t s_warp_above[kTopkThreads / 32], s_warp_gt[kTopkThreads / 32], s_warp_eq[kTopkThreads / 32];
  __shared__ uint32_t s_cta_gt[CL], s_cta_eq[CL];    // per CTA of the cluster: keys above / at T
  __shared__ uint32_t s_off[CL + 1];
  __shared__ uint32_t s_total, s_fast, s_Tb, s_Rb, s_out_before, s_eq_before;

  const int b = blockIdx.x / CL;
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  constexpr int kWarps = kTopkThreads / 32;
  const int k = p.k;
  griddep_wait();  // the scores come from the kernel before
  griddep_launch_dependents();
  if (p.clear && rank == 0 && tid == 0) p.clear[b] = 0;

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
  uint32_t* cand_key = sm_keys + p.cache_keys;
  uint32_t* gbuf = cand_key + kCandCap;
  uint16_t* wlists = (uint16_t*)(gbuf + kCandTotal);

  auto key_at = [&](int i) -> uint32_t {  // i relative to c0
    return cached ? sm_keys[i] : float_key(row[c0 + i]);
  };
  // keys i..i+3 (i a multiple of 4; entries at or beyond `end` are 0)
  auto key4 = [&](int i, int end, uint32_t* kq) {
    if (i + 3 < m) {
      if (cached) {
        const uint4 v = *(const uint4*)(sm_keys + i);
        kq[0] = v.x; kq[1] = v.y; kq[2] = v.z; kq[3] = v.w;
      } else {
        const float4 v = *(const float4*)(row + c0 + i);
        kq[0] = float_key(v.x); kq[1] = float_key(v.y); kq[2] = float_key(v.z); kq[3] = float_key(v.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) kq[e] = i + e < m ? key_at(i + e) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (i + e >= end) kq[e] = 0u;
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
    if (p.done) {
      __syncthreads();
      count_done(p.done + b);
    }
    return;  // no distributed shared memory was touched
  }

  // the histogram starts zeroed here; every radix pass leaves it zeroed again
  for (int d = tid; d < 2048; d += kTopkThreads) hist[d] = 0;
  if (cached) {
    // four 16-byte loads in flight per thread (indices clamped into the slice, so every
    // load is issued), then their keys into shared memory
    constexpr int kU = 4, kStep = kTopkThreads * 4;
    const int m4 = m & ~3;
    for (int i0 = tid * 4; i0 < m4; i0 += kStep * kU) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) v[u] = *(const float4*)(row + c0 + min(i0 + u * kStep, m4 - 4));
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * kStep;
        if (i < m4) *(uint4*)(sm_keys + i) = make_uint4(float_key(v[u].x), float_key(v[u].y), float_key(v[u].z), float_key(v[u].w));
      }
    }
    for (int i = m4 + tid; i < m; i += kTopkThreads) sm_keys[i] = float_key(row[c0 + i]);
  }

  // Find the bin (of `width` bits at `shift`) holding the k_rem-th largest key among the
  // keys whose bits above the digit equal `prefix`; bins scanned high to low.  With
  // `local`, only this CTA's `vals` are counted; otherwise the cluster's slices.  `hist` is
  // zero on entry and on exit: each thread clears the bins it read once no other CTA reads
  // them any more.
  uint32_t prefix = 0;
  uint32_t k_rem = (uint32_t)k;
  auto radix_pass = [&](int shift, int width, bool local, const uint32_t* vals, int nvals) {
    const int nbins = 1 << width;
    const uint32_t dmask = (uint32_t)nbins - 1u;
    const int hi_shift = shift + width;
    __syncthreads();  // the keys (and, in the first pass, the zeroed histogram) are in place
    // scores crowd into few bins, so lanes of a warp that hit the same bin add once
    auto count = [&](bool ok, uint32_t key) {
      if (ok) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    };
    if (vals) {
      for (int i0 = 0; i0 < nvals; i0 += kTopkThreads) {  // whole warps step together
        const int i = i0 + tid;
        const uint32_t key = i < nvals ? vals[i] : 0u;
        count(i < nvals && ((hi_shift >= 32) || ((key >> hi_shift) == prefix)), key);
      }
    } else {
      for (int i0 = 0; i0 < nvals; i0 += kTopkThreads * 4) {
        const int i = i0 + tid * 4;
        uint32_t kq[4];
        key4(i, nvals, kq);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          count(i + e < nvals && ((hi_shift >= 32) || ((kq[e] >> hi_shift) == prefix)), kq[e]);
      }
    }
    __syncthreads();
    const uint32_t* h_all = hist;
    if (!local) {
      cluster.sync();
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
      // no CTA reads this one's histogram any more: clear it for the next pass
      for (int d = tid; d < 2048; d += kTopkThreads) hist[d] = 0;
      // all of this thread's remote reads first (nbins <= 2048 = 4 per thread), then the stores
      uint32_t gv[2048 / kTopkThreads];
#pragma unroll
      for (int u = 0; u < 2048 / kTopkThreads; ++u) {
        const int d = tid + u * kTopkThreads;
        gv[u] = d < nbins ? cluster.map_shared_rank(red, d / slice)[d % slice] : 0u;
      }
#pragma unroll
      for (int u = 0; u < 2048 / kTopkThreads; ++u) {
        const int d = tid + u * kTopkThreads;
        if (d < nbins) ghist[d] = gv[u];
      }
      __syncthreads();
      h_all = ghist;
    }
    const int per = nbins / kTopkThreads;  // 4 or 2 bins per thread
    uint32_t hv[2048 / kTopkThreads];
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 2048 / kTopkThreads; ++j) {
      hv[j] = j < per ? h_all[nbins - 1 - (tid * per + j)] : 0u;
      mine += hv[j];
    }
    if (local) {  // this thread's bins are read: clear them for the next pass
#pragma unroll
      for (int j = 0; j < 2048 / kTopkThreads; ++j)
        if (j < per) hist[nbins - 1 - (tid * per + j)] = 0;
    }
    unsigned long long tot;
    uint32_t above = (uint32_t)block_excl_scan_u64(mine, scan_tmp, &tot);
#pragma unroll
    for (int j = 0; j < 2048 / kTopkThreads; ++j) {
      if (j < per) {
        const int d = nbins - 1 - (tid * per + j);
        if (above < k_rem && above + hv[j] >= k_rem) {
          s_found_bin = d;
          s_found_above = above;
        }
        above += hv[j];
      }
    }
    __syncthreads();
    // no barrier after these reads: the next write of s_found_* comes after the next pass's
    // counting barrier, which every thread reaches only after reading them
    prefix = (prefix << width) | (uint32_t)s_found_bin;
    k_rem -= s_found_above;
  };

  // ---- pass 0 over the whole request: the top 11 bits
  radix_pass(21, 11, false, nullptr, m);
  const uint32_t t0 = prefix;

  // ---- collect.  Each warp walks a contiguous segment of the slice (the one it emits
  // from) 32 keys at a time in position order and keeps, in order, the offsets of its
  // keys at or above bin t0 -- every output comes from these lists.  The keys of bin t0
  // (the only undecided ones) also go to the CTA's candidate buffer.
  const int seg = ((m + kWarps * 128 - 1) / (kWarps * 128)) * 128;
  const int i0 = min(m, warp * seg), i1 = min(m, i0 + seg);
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint16_t* wl = wlists + warp * kWarpList;
  if (tid == 0) {
    s_ncand = 0;
    s_overflow = seg > 65535 ? 1u : 0u;  // offsets are 16-bit
  }
  __syncthreads();
  uint32_t nl = 0;  // length of this warp's list
  {
    uint32_t nc = 0;  // keys of bin t0 in this warp's segment
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      const bool in = i < i1;
      const uint32_t key = in ? key_at(i) : 0u;
      const uint32_t bin = key >> 21;
      const bool sel = in && bin >= t0;
      const uint32_t selm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const uint32_t o = nl + __popc(selm & lt_mask);
        if (o < (uint32_t)kWarpList) wl[o] = (uint16_t)(i - i0);
      }
      nl += __popc(selm);
      nc += __popc(__ballot_sync(0xffffffffu, in && bin == t0));
    }
    // one reservation per warp, then the candidates straight from the (complete) list
    uint32_t cb = 0;
    if (lane == 0) {
      s_warp_above[warp] = nl - nc;
      if (nl > (uint32_t)kWarpList) s_overflow = 1;
      cb = atomicAdd(&s_ncand, nc);
    }
    cb = __shfl_sync(0xffffffffu, cb, 0);
    if (nl <= (uint32_t)kWarpList) {
      for (uint32_t jb = 0; jb < nl; jb += 32) {
        const uint32_t j = jb + lane;
        const uint32_t key = j < nl ? key_at(i0 + wl[j]) : 0u;
        const bool cand = j < nl && (key >> 21) == t0;
        const uint32_t cm = __ballot_sync(0xffffffffu, cand);
        if (cand) {
          const uint32_t o = cb + __popc(cm & lt_mask);
          if (o < (uint32_t)kCandCap) cand_key[o] = key;
        }
        cb += __popc(cm);
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t a = 0;
    for (int w = 0; w < kWarps; ++w) a += s_warp_above[w];
    s_nabove = a;
    if (s_ncand > (uint32_t)kCandCap) s_overflow = 1;
  }
  __syncthreads();
  cluster.sync();
  // lane c of warp 0 reads CTA c's counts: one distributed-shared-memory round trip;
  // every CTA reads the same values, so the choice of path is uniform over the cluster
  if (warp == 0) {
    uint32_t nc = 0, ov = 0, na = 0;
    if (lane < CL) {
      nc = *cluster.map_shared_rank(&s_ncand, lane);
      ov = *cluster.map_shared_rank(&s_overflow, lane);
      na = *cluster.map_shared_rank(&s_nabove, lane);
      s_cta_gt[lane] = na;  // keys above bin t0 (all above T), completed below
    }
    const uint32_t tot = __reduce_add_sync(0xffffffffu, nc);
    const bool anyov = __any_sync(0xffffffffu, ov != 0);
    uint32_t incl = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < CL) s_off[lane] = incl - nc;
    if (lane == 0) {
      s_off[CL] = tot;
      s_total = tot;
      s_fast = (!anyov && tot <= (uint32_t)kCandTotal) ? 1u : 0u;
    }
  }
  __syncthreads();
  const uint32_t total = s_total;
  const bool fast = s_fast != 0;

  uint32_t T, R, out_before, eq_before;
  unsigned long long pre;
  if (fast) {
    // every CTA brings all candidates (warp c from CTA c, eight loads in flight per lane)
    // and finishes the selection itself: the same T and counts everywhere, and no second
    // round of publishing and reading
    if (warp < CL) {
      const uint32_t* src = cluster.map_shared_rank(cand_key, warp);
      const uint32_t o = s_off[warp], cnt = s_off[warp + 1] - o;
      for (uint32_t jb = 0; jb < cnt; jb += 8 * 32) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t j = jb + u * 32 + lane;
          v[u] = j < cnt ? src[j] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t j = jb + u * 32 + lane;
          if (j < cnt) gbuf[o + j] = v[u];
        }
      }
    }
    __syncthreads();
    radix_pass(10, 11, true, gbuf, (int)total);
    radix_pass(0, 10, true, gbuf, (int)total);
    // warp c counts CTA c's candidates above the k-th key T and equal to it
    if (warp < CL) {
      const uint32_t o = s_off[warp], cnt = s_off[warp + 1] - o;
      uint32_t g = 0, e = 0;
      for (uint32_t j = lane; j < cnt; j += 32) {
        const uint32_t key = gbuf[o + j];
        g += key > prefix ? 1u : 0u;
        e += key == prefix ? 1u : 0u;
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
      if (lane == 0) {
        s_cta_gt[warp] += g;
        s_cta_eq[warp] = e;
      }
    }
    __syncthreads();
    if (warp == 0) {
      const uint32_t g = lane < CL ? s_cta_gt[lane] : 0u, e = lane < CL ? s_cta_eq[lane] : 0u;
      cluster_prefix(g, e, k_rem, rank, lane);
      if (lane == 0) {
        s_Tb = prefix;
        s_Rb = k_rem;
      }
    }
    __syncthreads();
    T = s_Tb;
    R = s_Rb;
    out_before = s_out_before;
    eq_before = s_eq_before;
    // per-warp counts over the warp's list, then their prefix over the CTA
    {
      uint32_t g = 0, e = 0;
      for (uint32_t j = lane; j < nl; j += 32) {
        const uint32_t key = key_at(i0 + wl[j]);
        g += key > T ? 1u : 0u;
        e += key == T ? 1u : 0u;
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
      if (lane == 0) {
        s_warp_gt[warp] = g;
        s_warp_eq[warp] = e;
      }
    }
    __syncthreads();
    const unsigned long long mine =
        lane == 0 ? (((unsigned long long)s_warp_gt[warp] << 32) | s_warp_eq[warp]) : 0ull;
    unsigned long long tot;
    const unsigned long long pre_t = block_excl_scan_u64(mine, scan_tmp, &tot);
    pre = __shfl_sync(0xffffffffu, pre_t, 0);
    // ---- emit from the list: ballots give every taken key its output slot (ties: lower
    // position first)
    const uint32_t eq_left = R > eq_before ? R - eq_before : 0u;  // ties this CTA may still take
    const uint32_t gt_pre = (uint32_t)(pre >> 32), eq_pre = (uint32_t)pre;
    uint32_t eq_seen = eq_pre;  // keys == T before this lane's current key, CTA-wide
    uint32_t out = out_before + gt_pre + min(eq_pre, eq_left);
    for (uint32_t jb = 0; jb < nl; jb += 32) {
      const uint32_t j = jb + lane;
      const bool in = j < nl;
      const int i = in ? i0 + wl[j] : 0;
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
  } else {
    // ---- general path (too many keys share bin t0): two more cluster-wide passes
    radix_pass(10, 11, false, nullptr, m);
    radix_pass(0, 10, false, nullptr, m);
    T = prefix;
    R = k_rem;
    uint32_t n_gt = 0, n_eq = 0;
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < i1 ? key_at(i) : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, i < i1 && key > T));
      n_eq += __popc(__ballot_sync(0xffffffffu, i < i1 && key == T));
    }
    const unsigned long long mine = lane == 0 ? (((unsigned long long)n_gt << 32) | n_eq) : 0ull;
    unsigned long long tot;
    const unsigned long long pre_t = block_excl_scan_u64(mine, scan_tmp, &tot);
    pre = __shfl_sync(0xffffffffu, pre_t, 0);
    if (tid == 0) cnt_pub = tot;
    __syncthreads();
    cluster.sync();
    if (warp == 0) {
      const unsigned long long v = lane < CL ? *cluster.map_shared_rank(&cnt_pub, lane) : 0ull;
      cluster_prefix((uint32_t)(v >> 32), (uint32_t)v, R, rank, lane);
    }
    __syncthreads();
    out_before = s_out_before;
    eq_before = s_eq_before;
    // ---- emit: each warp walks its segment 32 keys at a time in position order
    const uint32_t eq_left = R > eq_before ? R - eq_before : 0u;
    const uint32_t gt_pre = (uint32_t)(pre >> 32), eq_pre = (uint32_t)pre;
    uint32_t eq_seen = eq_pre;
    uint32_t out = out_before + gt_pre + min(eq_pre, eq_left);
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
  }
  if (p.thr && rank == 0 && tid == 0) p.thr[b] = key_float(T);
  if (p.done) {
    __syncthreads();
    count_done(p.done + b);
  }
  cluster.sync();  // keep this CTA's shared memory alive until the cluster is done with it
}

}  // namespace ls
