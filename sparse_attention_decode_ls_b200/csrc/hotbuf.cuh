// a4 / a5. Hot-buffer resolve and miss gather (XM-Sparse, hot-buffer section: HBM
// keeps a per-request hot KV buffer; after each step's sparse selection only the
// selected KV that misses it is fetched from the full history).
//
// hotbuf_resolve: one CTA per request.  Classifies each selection as hit (resident)
// or miss, compacts the misses in selection order, finds the n_miss first victims in
// the order (empty first, recent score, slot) by a radix select over 64-bit composite
// keys and ranks them by counting, hands the i-th victim to the i-th miss, and updates
// both maps and the recent scores in place.
//
// gather_misses: copies each missed 1,152-byte row from pinned host memory into its
// slot (or, in the decode step, into a staging row in miss order); every thread moves
// 16-byte vectors, and each warp keeps several rows' loads in flight so that the PCIe
// link, not latency, sets the pace.
//
// hotbuf_classify + copy_staged: the decode step's split of the same work.  The
// classify pass (which selections are resident, the misses in selection order) is all
// the host-link fetch needs, so the fetch starts into staging rows while the victim
// order is still being sorted; once both are done the staged rows are copied into
// their victim slots.
#pragma once
#include "common.cuh"

namespace ls {

struct HotbufParams {
  int B, k, n_slots, max_len;
  const int* sel;
  const float* sel_score;
  int* pos_of_slot;
  float* recent;
  int* slot_of_pos;
  int* sel_slot;
  int* miss_pos;
  int* miss_slot;
  int* n_miss;
};

constexpr int kHbThreads = 1024;
constexpr int kHbMaxSlots = 4096;
// dynamic shared memory of the resolve: keys (8 B), miss list (4 B), then the radix
// histogram (16 KB) overlaid by up to 4,096 victim keys (8 B)
constexpr int kHbResolveSmem = kHbMaxSlots * (8 + 4 + 8);

__global__ void __launch_bounds__(kHbThreads, 1) hotbuf_resolve_kernel(const HotbufParams p) {
  extern __shared__ unsigned long long keys[];       // [4096] victim keys, then the victim order
  int* miss_j = (int*)(keys + kHbMaxSlots);          // [4096] selection index of the i-th miss
  uint32_t* scratch = (uint32_t*)(miss_j + kHbMaxSlots);  // radix histogram, then victim keys
  __shared__ uint8_t pinned[kHbMaxSlots];
  __shared__ unsigned long long scan_tmp[32];
  __shared__ int s_sel_bin;
  __shared__ uint32_t s_sel_below, s_nvict;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int k = p.k, S = p.n_slots;
  const int* sel = p.sel + (size_t)b * k;
  int* pos_of_slot = p.pos_of_slot + (size_t)b * S;
  float* recent = p.recent + (size_t)b * S;
  int* slot_of_pos = p.slot_of_pos + (size_t)b * p.max_len;
  int* sel_slot = p.sel_slot + (size_t)b * k;

  for (int s = tid; s < S; s += kHbThreads) pinned[s] = 0;
  __syncthreads();
  // ---- classify (contiguous per-thread ranges keep selection order for the scan)
  const int per = (k + kHbThreads - 1) / kHbThreads;  // <= 4
  const int j0 = min(k, tid * per), j1 = min(k, j0 + per);
  uint32_t my_miss = 0;
  uint32_t miss_bits = 0;
  for (int j = j0; j < j1; ++j) {
    const int pos = sel[j];
    int slot = -1;
    bool is_miss = false;
    if (pos >= 0) {
      if (pos >= p.max_len) {
        flag(LS_DEV_BOUNDS);
      } else {
        slot = slot_of_pos[pos];
        if (slot >= S) {
          flag(LS_DEV_BOUNDS);
          slot = -1;
        } else if (slot >= 0) {
          pinned[slot] = 1;
        } else {
          is_miss = true;
        }
      }
    }
    sel_slot[j] = slot;
    if (is_miss) {
      miss_bits |= 1u << (j - j0);
      ++my_miss;
    }
  }
  unsigned long long total;
  const uint32_t mpre = (uint32_t)block_excl_scan_u64(my_miss, scan_tmp, &total);
  const int n_miss = (int)total;
  {
    uint32_t o = mpre;
    for (int j = j0; j < j1; ++j) {
      if (miss_bits >> (j - j0) & 1u) {
        miss_j[o] = j;
        p.miss_pos[(size_t)b * k + o] = sel[j];
        ++o;
      }
    }
  }
  // ---- victims: the n_miss smallest keys (class, recent-score key, slot), class 0 empty,
  // 1 occupied, 2 pinned; keys are distinct (the slot is in them).  A radix select (four
  // 12-bit digits) finds the n_miss-th smallest key; the keys up to it are gathered and each
  // one's rank among them (a count of the smaller ones) is its victim order.
  __syncthreads();
  for (int s = tid; s < S; s += kHbThreads) {
    unsigned long long key;
    if (pinned[s]) {
      key = (2ull << 44) | s;
    } else if (pos_of_slot[s] < 0) {
      key = (unsigned long long)s;
    } else {
      key = (1ull << 44) | ((unsigned long long)float_key(recent[s]) << 12) | (unsigned long long)s;
    }
    keys[s] = key;
  }
  unsigned long long thr = 0;  // the n_miss-th smallest key
  if (n_miss > 0) {
    uint32_t* hist = scratch;  // 4,096 bins
    unsigned long long prefix = 0;
    uint32_t m_rem = (uint32_t)n_miss;
    for (int dg = 3; dg >= 0; --dg) {
      const int shift = dg * 12;
      for (int d = tid; d < 4096; d += kHbThreads) hist[d] = 0;
      __syncthreads();
      for (int s = tid; s < S; s += kHbThreads) {
        const unsigned long long key = keys[s];
        if (dg == 3 || (key >> (shift + 12)) == prefix) atomicAdd(&hist[(key >> shift) & 4095ull], 1u);
      }
      __syncthreads();
      // bins in ascending order, four per thread
      uint32_t mine = hist[4 * tid] + hist[4 * tid + 1] + hist[4 * tid + 2] + hist[4 * tid + 3];
      unsigned long long tot;
      uint32_t below = (uint32_t)block_excl_scan_u64(mine, scan_tmp, &tot);
      for (int j = 0; j < 4; ++j) {
        const uint32_t h = hist[4 * tid + j];
        if (below < m_rem && below + h >= m_rem) {
          s_sel_bin = 4 * tid + j;
          s_sel_below = below;
        }
        below += h;
      }
      __syncthreads();
      prefix = (prefix << 12) | (unsigned long long)s_sel_bin;
      m_rem -= s_sel_below;
      __syncthreads();
    }
    thr = prefix;
    // the keys up to the threshold (exactly n_miss of them), then their ranks
    if (tid == 0) s_nvict = 0;
    __syncthreads();
    unsigned long long* vict = (unsigned long long*)hist;  // reuses the histogram space
    for (int s = tid; s < S; s += kHbThreads) {
      const unsigned long long key = keys[s];
      if (key <= thr) vict[atomicAdd(&s_nvict, 1u)] = key;
    }
    __syncthreads();
    const int nv = (int)s_nvict;  // == n_miss
    for (int i = tid; i < nv; i += kHbThreads) {
      const unsigned long long key = vict[i];
      int rank = 0;
      for (int j = 0; j < nv; ++j) rank += vict[j] < key ? 1 : 0;
      keys[rank] = key;  // the victim order, over the start of the key array
    }
    __syncthreads();
  }
  // ---- apply: the i-th miss takes the i-th victim
  for (int i = tid; i < n_miss; i += kHbThreads) {
    const unsigned long long key = keys[i];
    const int v = (int)(key & 0xFFFull);
    if ((key >> 44) >= 2ull) {  // ran out of unpinned slots
      flag(LS_DEV_CAPACITY);
      p.miss_slot[(size_t)b * k + i] = -1;
      continue;
    }
    const int pos = sel[miss_j[i]];
    const int old = pos_of_slot[v];
    if (old >= 0 && old < p.max_len) slot_of_pos[old] = -1;
    pos_of_slot[v] = pos;
    slot_of_pos[pos] = v;
    sel_slot[miss_j[i]] = v;
    p.miss_slot[(size_t)b * k + i] = v;
  }
  for (int i = n_miss + tid; i < k; i += kHbThreads) {
    p.miss_pos[(size_t)b * k + i] = -1;
    p.miss_slot[(size_t)b * k + i] = -1;
  }
  __syncthreads();
  for (int j = tid; j < k; j += kHbThreads) {
    const int s = sel_slot[j];
    if (s >= 0) recent[s] = p.sel_score[(size_t)b * k + j];
  }
  if (tid == 0) p.n_miss[b] = n_miss;
}

struct ClassifyParams {
  int B, k, n_slots, max_len;
  const int* sel;
  const int* slot_of_pos;
  int* hit_slot;   // [B,k] the slots of the resident selections in selection order, -1 after them
  int* n_hit;      // [B]
  int* miss_pos;   // [B,k] the missing positions in selection order, -1 after them
  int* miss_row;   // [B,k] i at the i-th miss, -1 after them (rows of the staging area)
  int* n_miss;     // [B]
};

// One CTA per request; the same classification as the resolve's first phase, without
// touching the maps.
__global__ void __launch_bounds__(kHbThreads, 1) hotbuf_classify_kernel(const ClassifyParams p) {
  __shared__ unsigned long long scan_tmp[32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int k = p.k, S = p.n_slots;
  const int* sel = p.sel + (size_t)b * k;
  const int* slot_of_pos = p.slot_of_pos + (size_t)b * p.max_len;
  const int per = (k + kHbThreads - 1) / kHbThreads;  // <= 4
  const int j0 = min(k, tid * per), j1 = min(k, j0 + per);
  int pos[4], slot[4];
  uint32_t n_m = 0, n_h = 0;
  // all of this thread's selections first, then all their map lookups: two round trips
#pragma unroll
  for (int q = 0; q < 4; ++q) pos[q] = j0 + q < j1 ? sel[j0 + q] : -1;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    slot[q] = -2;  // neither (padding or out of range)
    if (pos[q] >= 0) {
      if (pos[q] >= p.max_len) {
        flag(LS_DEV_BOUNDS);
      } else {
        slot[q] = slot_of_pos[pos[q]];
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (slot[q] >= S) {
      flag(LS_DEV_BOUNDS);
      slot[q] = -2;
    }
    n_m += slot[q] == -1;
    n_h += slot[q] >= 0;
  }
  // one scan of both counts: misses in the low half, hits in the high half
  unsigned long long total;
  const unsigned long long pre = block_excl_scan_u64(((unsigned long long)n_h << 32) | n_m, scan_tmp, &total);
  uint32_t om = (uint32_t)pre, oh = (uint32_t)(pre >> 32);
  for (int j = j0; j < j1; ++j) {
    const int q = j - j0;
    if (slot[q] == -1) {
      p.miss_pos[(size_t)b * k + om] = pos[q];
      p.miss_row[(size_t)b * k + om] = (int)om;
      ++om;
    } else if (slot[q] >= 0) {
      p.hit_slot[(size_t)b * k + oh] = slot[q];
      ++oh;
    }
  }
  const int n_miss = (int)(uint32_t)total, n_hit = (int)(total >> 32);
  for (int i = n_miss + tid; i < k; i += kHbThreads) {
    p.miss_pos[(size_t)b * k + i] = -1;
    p.miss_row[(size_t)b * k + i] = -1;
  }
  for (int i = n_hit + tid; i < k; i += kHbThreads) p.hit_slot[(size_t)b * k + i] = -1;
  if (tid == 0) {
    p.n_miss[b] = n_miss;
    p.n_hit[b] = n_hit;
  }
}

struct GatherParams {
  int B, k, n_slots, max_pages;
  long long row_bytes, num_pages;
  const char* host;
  const int* page_table;
  const int* miss_pos;
  const int* miss_slot;
  const int* n_miss;
  char* hbuf;
  char* stage;   // optional: the i-th miss goes to staging row b*k + i (miss_slot unused)
};

// grid (ctas_per_req, B), 128 threads and at most 64 registers each, so that a gather
// CTA fits beside an attention CTA on one SM.  A warp owns 2 rows at a time and issues
// all their 16-byte loads before storing any.
constexpr int kGatherThreads = 128;
__global__ void __launch_bounds__(kGatherThreads, 8) gather_misses_kernel(const GatherParams p) {
  const int b = blockIdx.y;
  const int warp = warp_id(), lane = lane_id();
  const int nm = p.n_miss[b];
  if (nm < 0 || nm > p.k) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  const int chunks = (int)(p.row_bytes >> 4);
  constexpr int kWarps = kGatherThreads / 32;
  const int gw = blockIdx.x * kWarps + warp, nw = gridDim.x * kWarps;
  constexpr int R = 2;
  for (int i0 = gw * R; i0 < nm; i0 += nw * R) {
    const char* src[R];
    char* dst[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      src[q] = nullptr;
      dst[q] = nullptr;
      const int i = i0 + q;
      if (i < nm) {
        const int pos = p.miss_pos[(size_t)b * p.k + i];
        const int slot = p.stage ? 0 : p.miss_slot[(size_t)b * p.k + i];
        const int lp = pos >> 6;
        if (pos >= 0 && lp < p.max_pages && slot >= 0 && slot < p.n_slots) {
          const int page = p.page_table[(size_t)b * p.max_pages + lp];
          if (page >= 0 && page < p.num_pages) {
            src[q] = p.host + ((long long)page * 64 + (pos & 63)) * p.row_bytes;
            dst[q] = p.stage ? p.stage + ((long long)b * p.k + i) * p.row_bytes
                             : p.hbuf + ((long long)b * p.n_slots + slot) * p.row_bytes;
          } else {
            flag(LS_DEV_BOUNDS);
          }
        } else {
          flag(LS_DEV_BOUNDS);
        }
      }
    }
    for (int c0 = 0; c0 < chunks; c0 += 32 * 3) {
      uint4 v[R][3];
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int e = 0; e < 3; ++e) {
          const int c = c0 + e * 32 + lane;
          if (src[q] && c < chunks) v[q][e] = *(const uint4*)(src[q] + (size_t)c * 16);
        }
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int e = 0; e < 3; ++e) {
          const int c = c0 + e * 32 + lane;
          if (dst[q] && c < chunks) *(uint4*)(dst[q] + (size_t)c * 16) = v[q][e];
        }
    }
  }
}

// Prefill: a hot buffer seeded with each request's most recent n_slots positions (slot
// s holds p = L - n_slots + s when p >= 0), recent scores 0, and the list of seeded
// (position, slot) pairs for the row gather.  grid (x, B), 256 threads: the grid strides
// over slot_of_pos; CTA 0 of each request also writes the slot side and the lists.
struct SeedParams {
  int B, n_slots, max_len, max_pages;
  const int* lens;
  int* pos_of_slot;  // [B,n_slots]
  int* slot_of_pos;  // [B,max_len]
  float* recent;     // [B,n_slots]
  int* seed_pos;     // [B,n_slots] positions in slot order, -1 after them
  int* seed_slot;    // [B,n_slots]
  int* seed_n;       // [B]
};

__global__ void __launch_bounds__(256) seed_hotbuf_kernel(const SeedParams p) {
  const int b = blockIdx.y;
  const int L = p.lens[b], S = p.n_slots;
  if (L < 0 || L > p.max_len || L > p.max_pages * 64) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      flag(LS_DEV_BOUNDS);
      p.seed_n[b] = 0;
    }
    return;
  }
  const int first = L - S;  // position held by slot 0 (may be negative: empty slots)
  for (int q = blockIdx.x * 256 + threadIdx.x; q < p.max_len; q += gridDim.x * 256)
    p.slot_of_pos[(size_t)b * p.max_len + q] = (q < L && q >= first) ? q - first : -1;
  if (blockIdx.x != 0) return;
  const int s0 = max(0, -first);  // first non-empty slot
  for (int s = threadIdx.x; s < S; s += 256) {
    const int pos = first + s;
    p.pos_of_slot[(size_t)b * S + s] = pos >= 0 ? pos : -1;
    p.recent[(size_t)b * S + s] = 0.f;
    const int i = s - s0;  // the gather lists, in slot order
    if (s >= s0) {
      p.seed_pos[(size_t)b * S + i] = pos;
      p.seed_slot[(size_t)b * S + i] = s;
    }
    if (s >= S - s0) {  // the tail of the lists past the seeded entries
      p.seed_pos[(size_t)b * S + s] = -1;
      p.seed_slot[(size_t)b * S + s] = -1;
    }
  }
  if (threadIdx.x == 0) p.seed_n[b] = S - s0;
}

struct StageCopyParams {
  int B, k, n_slots;
  long long row_bytes;
  const char* stage;     // [B,k,row_bytes]: the i-th miss of request b at row b*k + i
  const int* miss_slot;  // [B,k] the i-th miss's victim slot (-1: none)
  const int* n_miss;     // [B]
  char* hbuf;            // [B,n_slots,row_bytes]
};

// grid (ctas_per_req, B), 256 threads: a warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) copy_staged_kernel(const StageCopyParams p) {
  const int b = blockIdx.y;
  const int nm = p.n_miss[b];
  if (nm < 0 || nm > p.k) return;  // the resolve has flagged it
  const int chunks = (int)(p.row_bytes >> 4);
  const int gw = blockIdx.x * 8 + warp_id(), nw = gridDim.x * 8, lane = lane_id();
  for (int i = gw; i < nm; i += nw) {
    const int slot = p.miss_slot[(size_t)b * p.k + i];
    if (slot < 0 || slot >= p.n_slots) continue;  // out of capacity: flagged by the resolve
    const uint4* src = (const uint4*)(p.stage + ((long long)b * p.k + i) * p.row_bytes);
    uint4* dst = (uint4*)(p.hbuf + ((long long)b * p.n_slots + slot) * p.row_bytes);
    for (int c = lane; c < chunks; c += 32) dst[c] = src[c];
  }
}

}  // namespace ls
