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
  int smem_bytes;            // dynamic shared memory of the launch
  int* clear;                // optional [B]: set to 0 (a per-request count the next kernel of
                             //   the step adds up; see AttnParams::done)
  int* done;                 // optional [B], zero at launch: every CTA adds 1 once its outputs
                             //   are stored (see AttnParams::ready)
  // optional: the indexer's candidate lists (see the candidate filter in index_score.cuh)
  int* filt;                 // [B][kFiltInts]: read, then zeroed for the next step
  const int* cand_cnt;       // [B][cand_lists] candidates per list (one per indexer epilogue warp)
  const int* cand_pos;       // [B][cand_lists][kCandPerWarp]
  const float* cand_score;
  int cand_lists;            // the indexer's lists per request
  // optional, with the candidate lists: the attention's paged rows, which the CTAs other than
  // CTA 0 bring into L2 (bulk prefetch) while CTA 0 selects
  const uint8_t* pf_rows;    // row r at pf_rows + r * pf_row_bytes, pf_bytes of it fetched
  const int* pf_pt;          // [B][pf_max_pages] page table (row = page * 64 + position % 64)
  int pf_max_pages;
  long long pf_num_rows;
  long long pf_row_bytes;
  int pf_bytes;
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


constexpr int kFastMaxCand = 6144;  // candidates the candidate path holds
constexpr int kFastBins = 4096;     // histogram bins (12 bits of a key at a time)
constexpr int kFastShift = 12;      // first pass: bins of 2^12 keys above key(tau), the last open
constexpr int kFastList = 64;       // keys in the k-th key's bin that the list rank takes

__host__ __device__ constexpr int fast_round(int x, int m) { return (x + m - 1) / m * m; }
// Shared memory (bytes) the candidate path needs for a request of L positions and n
// candidates: their keys and positions, a bitmap of the chosen positions and a room that
// holds the histogram, then the bitmap words' prefix counts (or, on the general route, the
// bitmap of the keys equal to the k-th).
__host__ __device__ constexpr int fast_smem_bytes(int L, int n) {
  return (fast_round(2 * n, 4) + fast_round((L + 31) / 32, 8) +
          (fast_round((L + 31) / 32, 8) > kFastBins ? fast_round((L + 31) / 32, 8) : kFastBins)) * 4;
}

// The top-k of one request from the indexer's candidate lists (every key of the top k is
// among them, see TopkParams::filt), by one CTA of kTopkThreads threads.  coff[c] is where
// list c starts (coff[lists] = n); list: 2 * kFastList words of shared scratch.
//  1. Each candidate is loaded (eight per thread in flight) and counted in the bin of
//     (key - key(tau)) >> 12 (the candidates crowd just above tau: bins measured from there
//     spread them; the last bin is open-ended).
//  2. One scan of the bins from the top finds the bin tb of the k-th largest key.
//  3. Every key in a higher bin is chosen; bin tb's keys go to a list, where each is ranked
//     exactly (larger key first, then lower position) and the first k - (keys above tb) are
//     chosen.  A bin too crowded for the list (many equal keys) takes the general route: the
//     k-th largest key T by a radix pass over the low 12 bits of bin tb's keys (over whole keys,
//     12 bits at a time, for the open last bin), then the keys equal to T in a bitmap, of which
//     the lowest-positioned are taken.
//  4. A bitmap holds the chosen positions; from its words' prefix counts each chosen candidate
//     writes its own slot, so the positions leave in ascending order.  Its score is its key
//     read back as a float: the same bits the indexer stored in the score row.
__device__ __forceinline__ void topk_from_candidates(const TopkParams& p, int b, int L, int n, uint32_t* smem,
                                                     const int* coff, uint32_t* list, uint32_t* scan32,
                                                     uint32_t* s_misc, uint32_t tau_bits) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = p.k, nl = p.cand_lists, nw8 = fast_round((L + 31) >> 5, 8);
  uint32_t* keys = smem;
  int* cpos = (int*)(keys + n);
  uint32_t* bits = smem + fast_round(2 * n, 4);  // 16-byte aligned
  uint32_t* room = bits + nw8;
  uint32_t* lkey = list;
  int* lpos = (int*)(list + kFastList);
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  for (int w = tid * 4; w < kFastBins; w += kTopkThreads * 4) *(uint4*)(room + w) = z4;
  if (tid == 0) {
    s_misc[1] = 0u;         // keys in the list
    s_misc[2] = kFastBins;  // the k-th key's bin (none yet)
  }
  const uint32_t tk = float_key(__uint_as_float(tau_bits));
  __syncthreads();
  // ---- 1. load and count: warp w takes lists w, w + 16, ..., ten at a time (lane j entry
  // j; a list longer than 32 entries takes more turns), all their loads in flight at once
  const size_t base = (size_t)b * nl * kCandPerWarp;
  constexpr int kW = kTopkThreads / 32;
  auto take = [&](float sc, int ps, int at) {
    const uint32_t key = float_key(sc);
    keys[at] = key;
    cpos[at] = ps;
    if (key >= tk) atomicAdd(&room[min((key - tk) >> kFastShift, (uint32_t)(kFastBins - 1))], 1u);
  };
  constexpr int kPer = 10;  // 16 warps x 10: the 148 lists of a 37-CTA indexer in one round
  for (int l0 = warp; l0 < nl; l0 += kPer * kW) {
    float sq[kPer];
    int pq[kPer], at[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int l = l0 + u * kW;
      at[u] = -1;
      if (l < nl) {
        const int o = coff[l], c = min(coff[l + 1] - o, kCandPerWarp);
        if (lane < c) {
          const size_t src = base + (size_t)l * kCandPerWarp + lane;
          sq[u] = p.cand_score[src];
          pq[u] = p.cand_pos[src];
          at[u] = o + lane;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u)
      if (at[u] >= 0) take(sq[u], pq[u], at[u]);
    for (int u = 0; u < kPer; ++u) {  // entries 32 and up (a rare long list)
      const int l = l0 + u * kW;
      if (l >= nl) break;
      const int o = coff[l], c = min(coff[l + 1] - o, kCandPerWarp);
      for (int j = 32 + lane; j < c; j += 32) {
        const size_t src = base + (size_t)l * kCandPerWarp + j;
        take(p.cand_score[src], p.cand_pos[src], o + j);
      }
    }
  }
  __syncthreads();
  // ---- 2. the k-th key's bin: thread t reads bins [4088 - 8t, 4095 - 8t] from the top
  {
    constexpr int per = kFastBins / kTopkThreads;
    static_assert(per == 8, "eight bins per thread");
    const int top = kFastBins - per * (tid + 1);
    const uint4 a = *(const uint4*)(room + top), c = *(const uint4*)(room + top + 4);
    const uint32_t h[per] = {c.w, c.z, c.y, c.x, a.w, a.z, a.y, a.x};
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) mine += h[j];
    uint32_t tot;
    uint32_t above = block_excl_scan_u32(mine, scan32, &tot);
#pragma unroll
    for (int j = 0; j < per; ++j) {
      if (above < (uint32_t)k && above + h[j] >= (uint32_t)k) {
        s_misc[2] = (uint32_t)(top + per - 1 - j);
        s_misc[3] = above;
      }
      above += h[j];
    }
  }
  __syncthreads();
  const uint32_t tb = s_misc[2], r0 = (uint32_t)k - s_misc[3];  // r0 of bin tb's keys are chosen
  for (int w = tid * 4; w < nw8; w += kTopkThreads * 4) *(uint4*)(bits + w) = z4;
  __syncthreads();
  // ---- 3. keys above bin tb chosen, bin tb's keys listed
  for (int i = tid; i < n; i += kTopkThreads) {
    const uint32_t key = keys[i];
    const int ps = cpos[i];
    if (key < tk || ps < 0 || ps >= L) continue;
    const uint32_t bin = min((key - tk) >> kFastShift, (uint32_t)(kFastBins - 1));
    if (bin > tb) {
      atomicOr(&bits[ps >> 5], 1u << (ps & 31));
    } else if (bin == tb) {
      const uint32_t o = atomicAdd(&s_misc[1], 1u);
      if (o < (uint32_t)kFastList) {
        lkey[o] = key;
        lpos[o] = ps;
      }
    }
  }
  __syncthreads();
  const uint32_t m = s_misc[1];
  if (tb < (uint32_t)kFastBins && m <= (uint32_t)kFastList) {
    for (int e = tid; e < (int)m; e += kTopkThreads) {
      const uint32_t ke = lkey[e];
      const int pe = lpos[e];
      uint32_t r = 0;
      for (int j = 0; j < (int)m; ++j) {
        const uint32_t kj = lkey[j];
        r += (kj > ke || (kj == ke && lpos[j] < pe)) ? 1u : 0u;
      }
      if (r < r0) atomicOr(&bits[pe >> 5], 1u << (pe & 31));
    }
  } else {
    // the general route: T and R by radix passes over d = key - base from bit hi down, among
    // the keys whose bits above hi equal prefix: the low 12 bits of bin tb, or whole keys
    constexpr int per = kFastBins / kTopkThreads;
    const bool open = tb >= (uint32_t)(kFastBins - 1);
    const uint32_t base = open ? 0u : tk;
    uint32_t prefix = open ? 0u : tb, k_rem = open ? (uint32_t)k : r0;
    for (int hi = open ? 32 : kFastShift; hi > 0;) {
      const int width = min(12, hi), shift = hi - width;
      const uint32_t nb = 1u << width;
      for (int d = tid; d < kFastBins; d += kTopkThreads) room[d] = 0u;
      __syncthreads();
      for (int i = tid; i < n; i += kTopkThreads) {
        const uint32_t key = keys[i], d = key - base;
        if (key >= base && (hi >= 32 || (d >> hi) == prefix)) atomicAdd(&room[(d >> shift) & (nb - 1u)], 1u);
      }
      __syncthreads();
      uint32_t h[per], mine = 0;
#pragma unroll
      for (int j = 0; j < per; ++j) {
        const int bin = (int)nb - 1 - (tid * per + j);
        h[j] = bin >= 0 ? room[bin] : 0u;
        mine += h[j];
      }
      uint32_t tot;
      uint32_t above = block_excl_scan_u32(mine, scan32, &tot);
#pragma unroll
      for (int j = 0; j < per; ++j) {
        if (above < k_rem && above + h[j] >= k_rem) {
          s_misc[2] = (uint32_t)((int)nb - 1 - (tid * per + j));
          s_misc[3] = above;
        }
        above += h[j];
      }
      __syncthreads();
      prefix = (prefix << width) | s_misc[2];
      k_rem -= s_misc[3];
      hi = shift;
      __syncthreads();
    }
    const uint32_t T = base + prefix, R = k_rem;  // every key > T, and the R lowest-positioned == T
    uint32_t* tbits = room;
    for (int w = tid; w < nw8; w += kTopkThreads) tbits[w] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const int ps = cpos[i];
      if (ps < 0 || ps >= L) continue;
      if (keys[i] > T) {
        atomicOr(&bits[ps >> 5], 1u << (ps & 31));
      } else if (keys[i] == T) {
        atomicOr(&tbits[ps >> 5], 1u << (ps & 31));
      }
    }
    __syncthreads();
    const int wpt = (nw8 + kTopkThreads - 1) / kTopkThreads;
    const int w0 = min(nw8, tid * wpt), w1 = min(nw8, w0 + wpt);
    uint32_t c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(tbits[w]);
    uint32_t tot;
    uint32_t seen = block_excl_scan_u32(c, scan32, &tot);
    for (int w = w0; w < w1 && seen < R; ++w) {
      uint32_t mm = tbits[w], take = 0u;
      while (mm && seen < R) {
        take |= mm & (~mm + 1u);  // lowest set bit
        mm &= mm - 1u;
        ++seen;
      }
      if (take) atomicOr(&bits[w], take);
    }
  }
  __syncthreads();
  // ---- 4. the words' prefix counts (in the room), then every chosen candidate's slot
  {
    const int wpt = fast_round((nw8 + kTopkThreads - 1) / kTopkThreads, 4);
    const int w0 = min(nw8, tid * wpt), w1 = min(nw8, w0 + wpt);
    uint32_t c = 0;
    for (int w = w0; w < w1; w += 4) {
      const uint4 v = *(const uint4*)(bits + w);
      c += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    }
    uint32_t tot;
    uint32_t o = block_excl_scan_u32(c, scan32, &tot);
    for (int w = w0; w < w1; w += 4) {
      const uint4 v = *(const uint4*)(bits + w);
      uint4 q;
      q.x = o;
      o += __popc(v.x);
      q.y = o;
      o += __popc(v.y);
      q.z = o;
      o += __popc(v.z);
      q.w = o;
      o += __popc(v.w);
      *(uint4*)(room + w) = q;
    }
    if (tid == 0 && tot != (uint32_t)k) flag(LS_DEV_BOUNDS);  // cannot happen: exactly k chosen
  }
  __syncthreads();
  const int off = p.pos_offset ? p.pos_offset[b] : 0;
  for (int i = tid; i < n; i += kTopkThreads) {
    const int ps = cpos[i];
    if (ps < 0 || ps >= L) continue;
    const uint32_t word = bits[ps >> 5], bit = 1u << (ps & 31);
    if (!(word & bit)) continue;
    const uint32_t o = room[ps >> 5] + __popc(word & (bit - 1u));
    if (o < (uint32_t)k) {
      if (p.idx) p.idx[(size_t)b * k + o] = ps + off;
      if (p.sel) p.sel[(size_t)b * k + o] = key_float(keys[i]);
    }
  }
}

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

  if (p.filt) {
    // The candidate path: when the indexer's lists for this request are complete, hold at
    // least k candidates and fit this CTA's shared memory, CTA 0 selects from them alone and
    // the other CTAs leave at once.  Every CTA reads the same words, so the choice is the same
    // in the whole cluster (and no distributed shared memory has been touched).  Warp 0 adds
    // up the lists' lengths into their offsets (in ghist), warp 1 reads the filter's state.
    const int* f = p.filt + (size_t)b * kFiltInts;
    int* coff = (int*)ghist;
    if (warp == 0) {
      // lane j adds up lists [8j, 8j + 8) of each 256, their counts loaded together
      const int nl = p.cand_lists;
      const int* cnt = p.cand_cnt + (size_t)b * nl;
      uint32_t run = 0;
      for (int c0 = 0; c0 < nl; c0 += 256) {
        uint32_t v[8], mine = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int l = c0 + lane * 8 + e;
          v[e] = l < nl ? (uint32_t)max(cnt[l], 0) : 0u;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) mine += v[e];
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t at = run + incl - mine;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int l = c0 + lane * 8 + e;
          if (l < nl) coff[l] = (int)at;
          at += v[e];
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        coff[nl] = (int)run;
        s_total = run;
      }
    } else if (warp == 1 && lane == 0) {
      s_fast = (f[kFiltReady] != 0 && f[kFiltIncomplete] == 0) ? 1u : 0u;
      s_Tb = (uint32_t)f[kFiltTau];  // the threshold's bits (s_Tb is the cluster path's, later)
    }
    const long long L0 = ((long long)p.lens[b] * p.len_mul + p.len_div - 1) / p.len_div;
    __syncthreads();
    const int nc = (int)s_total;
    const int Lq = (L0 < 0 || L0 > p.len_limit) ? 0 : (int)L0;
    const bool use = s_fast != 0 && nc >= k && nc <= kFastMaxCand && Lq > 0 && p.cand_lists < 2048 &&
                     fast_smem_bytes(Lq, nc) <= p.smem_bytes && !p.unit_list && !p.pos_list && !p.thr;
    // once every CTA of the cluster has read the request's words, CTA 0 zeroes them for the
    // next step (arrive now, wait when done: the candidate path does not wait for the others)
    cluster_arrive();
    if (use) {
      if (rank == 0) {
        topk_from_candidates(p, b, Lq, nc, sm_keys, coff, hist, (uint32_t*)scan_tmp, s_off, s_Tb);
        if (p.done) {
          __syncthreads();
          count_done(p.done + b, CL);  // counts for the whole cluster
        }
      } else if (p.pf_rows) {
        // the candidates' attention rows into L2 while CTA 0 selects (the HBM is idle then):
        // each warp of CTAs 1 .. CL-1 one list, one lane per entry
        const size_t lbase = (size_t)b * p.cand_lists * kCandPerWarp;
        for (int l = (rank - 1) * kWarps + warp; l < p.cand_lists; l += (CL - 1) * kWarps) {
          const int o = coff[l], c = min(coff[l + 1] - o, kCandPerWarp);
          for (int j = lane; j < c; j += 32) {
            const int ps = p.cand_pos[lbase + (size_t)l * kCandPerWarp + j];
            if (ps < 0 || ps >= Lq || (ps >> 6) >= p.pf_max_pages) continue;
            const int pg = p.pf_pt[(size_t)b * p.pf_max_pages + (ps >> 6)];
            const long long row = (long long)pg * 64 + (ps & 63);
            if (pg < 0 || row >= p.pf_num_rows) continue;
            prefetch_l2_bulk(p.pf_rows + row * p.pf_row_bytes, (uint32_t)p.pf_bytes);
          }
        }
      }
      cluster_wait();
      if (rank == 0 && tid < kFiltInts) p.filt[(size_t)b * kFiltInts + tid] = 0;
      return;  // no distributed shared memory was touched
    }
    cluster_wait();
    if (rank == 0 && tid < kFiltInts) p.filt[(size_t)b * kFiltInts + tid] = 0;
    __syncthreads();  // the fallback reuses ghist
  }

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
