// a6. Sparse attention over the selected rows only (LeanSparse, abstract: sparse
// attention limits the history read by each query).
//
//   s_j = scale * q_h . K_j,  o_h = sum_j softmax(s)_j V_j,  lse_h = log sum_j exp(s_j)
//
// * attn_mla_tc: MLA-absorbed decode, 128 query heads against one 576-wide latent KV
//   head whose first 512 dims are V, bf16, on tcgen05 tensor cores.
//     - Heads are the MMA M dimension (128); a tile of 64 selected rows is N.
//     - S = Q K^T (K = 576) and O += P V are tcgen05.mma kind::f16 with f32 TMEM
//       accumulators.  O for all 512 V dims would fill the whole 512-column TMEM, so a
//       pair of CTAs (a 2-CTA cluster) shares each (request, KV split): rank r keeps the
//       256-wide half O_r in TMEM and contracts S only over its own latent dims (its four
//       V panels and half of the K-only panel 8); the two 128 x 64 partials are swapped
//       through distributed shared memory and added, identically, on both sides.
//     - TMEM: O half (256 columns), two S tiles (2 x 64; P, as bf16 pairs, is written
//       over the first half of its own S tile), four Q panels (128).  Q panel 8 stays in
//       shared memory as the A operand of its K steps.
//     - Rows are gathered through the page table or the hot-buffer slots by TMA
//       tile::gather4 (four rows x one 128-byte panel per load, 128-byte swizzle) into a
//       three-stage ring; the same panels serve as the K-major B operand of S and the
//       MN-major B operand of PV.
//     - Online softmax in the exp2 domain with lazy rescaling (O is only rescaled
//       when the running max grows by more than 2^8).
//     - Split-KV across CTA pairs (enough to fill the GPU at small batch), merged by
//       attn_combine with the log-sum-exp rule.
// * attn_simt: CUDA-core kernel for fp32 (and a bf16 cross-check variant).
#pragma once
#include "common.cuh"

namespace ls {

struct AttnParams {
  int B, H, dk, dv, k;
  float scale;       // softmax scale (natural-log domain)
  int addressing;    // LS_ROWS_PAGED / LS_ROWS_SLOTS
  int max_pages, n_slots;
  long long row_stride, num_rows;
  const void* q;
  const void* krows;
  const void* vrows;
  const int* page_table;
  const int* sel;
  void* o;
  float* lse;
  int nsplit;
  float* part_o;     // [B,nsplit,dv/4,H,4] unnormalised partial outputs (4-dim granules, head next)
  float* part_ml;    // [B,nsplit,H,2] running max (log2 domain) and sum
  int split_base;    // tensor-core kernel: this launch's splits are partial slots
  int nsplit_total;  //   [split_base, split_base + nsplit) of nsplit_total per request
  int compacted;     // the valid entries of every request's selection come first
  int o_f32;         // tensor-core kernel: o is float32 (else bf16)
  const int* n_valid;  // optional [B]: and there are n_valid[b] of them; the splits share
                       //   those rows instead of all k entries
  const int* ready;    // optional [B]: the selection of request b is complete once ready[b]
  int ready_want;      //   reaches ready_want (the top-k's CTAs per request count themselves);
                       //   waited for per request instead of the whole kernel before
  int* done;           // optional [B], zero at launch: every CTA adds 1 once its split partial
                       //   is stored, and attn_combine starts on a request as soon as all
                       //   2 * nsplit of its CTAs have, instead of after the whole grid
  int merge;           // tensor-core kernel: the CTAs of all splits of a request form one
                       //   cluster and merge the splits in distributed shared memory (no
                       //   partials in global memory, no combine kernel); nsplit in {2, 4, 8}
};

// 2^x with the hardware approximation (relative error about 2^-22; results below the
// smallest normal flush to zero, which the softmax weights tolerate).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Row index of selection value sv of request b, or -1 (padding or out of range).
__device__ __forceinline__ long long attn_row(const AttnParams& p, int b, int sv) {
  if (sv < 0) return -1;
  long long row;
  if (p.addressing == LS_ROWS_PAGED) {
    const int lp = sv >> 6;
    if (lp >= p.max_pages) { flag(LS_DEV_BOUNDS); return -1; }
    const int page = p.page_table[(size_t)b * p.max_pages + lp];
    if (page < 0) { flag(LS_DEV_BOUNDS); return -1; }
    row = (long long)page * 64 + (sv & 63);
  } else {
    if (sv >= p.n_slots) { flag(LS_DEV_BOUNDS); return -1; }
    row = (long long)b * p.n_slots + sv;
  }
  if (row >= p.num_rows) { flag(LS_DEV_BOUNDS); return -1; }
  return row;
}

// =====================================================================================
// CUDA-core kernel: one (request, head) per CTA.
// =====================================================================================
template <bool BF16>
__global__ void __launch_bounds__(256) attn_simt(const AttnParams p) {
  extern __shared__ __align__(16) float sm_a[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  float* qs = sm_a;                       // [dk]
  float* s = qs + ((p.dk + 1) & ~1);      // [k]
  long long* rows = (long long*)(s + ((p.k + 1) & ~1));  // [k], 8-byte aligned
  __shared__ float red[32];
  using T = typename std::conditional<BF16, __nv_bfloat16, float>::type;
  const T* q = (const T*)p.q + ((size_t)b * p.H + h) * p.dk;
  for (int d = tid; d < p.dk; d += 256) qs[d] = (float)q[d];
  for (int j = tid; j < p.k; j += 256) rows[j] = attn_row(p, b, p.sel[(size_t)b * p.k + j]);
  __syncthreads();
  const T* K = (const T*)p.krows;
  const T* V = (const T*)p.vrows;
  // four-element vector loads when every row starts on a 4-element boundary
  const bool vec = (p.row_stride % 4) == 0 && (((uintptr_t)K | (uintptr_t)V) % (4 * sizeof(T))) == 0;
  // scores: a thread per selected row computes its whole dot product (all of the row's
  // loads in flight at once)
  for (int j = tid; j < p.k; j += 256) {
    const long long r = rows[j];
    float sc = -INFINITY;
    if (r >= 0) {
      const T* kr = K + r * p.row_stride;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      int d = 0;
      if (vec) {
        for (; d + 3 < p.dk; d += 4) {
          float x0, x1, x2, x3;
          if (BF16) {
            const uint2 u = *(const uint2*)(kr + d);
            x0 = __uint_as_float(u.x << 16); x1 = __uint_as_float(u.x & 0xFFFF0000u);
            x2 = __uint_as_float(u.y << 16); x3 = __uint_as_float(u.y & 0xFFFF0000u);
          } else {
            const float4 v = *(const float4*)(kr + d);
            x0 = v.x; x1 = v.y; x2 = v.z; x3 = v.w;
          }
          a0 = fmaf(qs[d], x0, a0); a1 = fmaf(qs[d + 1], x1, a1);
          a2 = fmaf(qs[d + 2], x2, a2); a3 = fmaf(qs[d + 3], x3, a3);
        }
      }
      for (; d < p.dk; ++d) a0 = fmaf(qs[d], (float)kr[d], a0);
      sc = ((a0 + a1) + (a2 + a3)) * p.scale;
    }
    s[j] = sc;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int j = tid; j < p.k; j += 256) mx = fmaxf(mx, s[j]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < p.k; j += 256) {
    const float e = rows[j] >= 0 ? expf(s[j] - mx) : 0.f;
    s[j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  float l = 0.f;
  for (int w = 0; w < 8; ++w) l += red[w];
  T* o = (T*)p.o + ((size_t)b * p.H + h) * p.dv;
  // output: warp w sums rows j = w (mod 8), lane c a group of four dims (one 512-byte
  // piece of a row per warp instruction); the eight warps' sums meet in shared memory
  __shared__ float4 part[8][32];
  const int ng = (p.dv + 3) / 4;
  for (int g0 = 0; g0 < ng; g0 += 32) {
    const int g = g0 + lane, d0 = 4 * g;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (g < ng) {
#pragma unroll 4
      for (int j = warp; j < p.k; j += 8) {
        const long long r = rows[j];
        const float w = r >= 0 ? s[j] : 0.f;
        const T* vr = V + (r >= 0 ? r : 0) * p.row_stride + d0;  // a skipped row reads row 0
        float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
        if (vec && d0 + 3 < p.dv) {
          if (BF16) {
            const uint2 u = *(const uint2*)vr;
            x0 = __uint_as_float(u.x << 16); x1 = __uint_as_float(u.x & 0xFFFF0000u);
            x2 = __uint_as_float(u.y << 16); x3 = __uint_as_float(u.y & 0xFFFF0000u);
          } else {
            const float4 v = *(const float4*)vr;
            x0 = v.x; x1 = v.y; x2 = v.z; x3 = v.w;
          }
        } else {
          x0 = (float)vr[0];
          if (d0 + 1 < p.dv) x1 = (float)vr[1];
          if (d0 + 2 < p.dv) x2 = (float)vr[2];
          if (d0 + 3 < p.dv) x3 = (float)vr[3];
        }
        if (r < 0) x0 = x1 = x2 = x3 = 0.f;  // a skipped row adds nothing, whatever row 0 holds
        acc.x = fmaf(w, x0, acc.x); acc.y = fmaf(w, x1, acc.y);
        acc.z = fmaf(w, x2, acc.z); acc.w = fmaf(w, x3, acc.w);
      }
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && g < ng) {
      float4 t = part[0][lane];
      for (int w = 1; w < 8; ++w) {
        const float4 u = part[w][lane];
        t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float vals[4] = {t.x * inv, t.y * inv, t.z * inv, t.w * inv};
      for (int e = 0; e < 4 && d0 + e < p.dv; ++e) o[d0 + e] = (T)vals[e];
    }
    __syncthreads();
  }
  if (tid == 0) p.lse[(size_t)b * p.H + h] = l > 0.f ? mx + logf(l) : -INFINITY;
}

// =====================================================================================
// tcgen05 MLA kernel
// =====================================================================================
namespace mla {
constexpr int H = 128, DK = 576, DV = 512, DVH = 256, N = 64;  // N: selected rows per tile
constexpr int kPanels = DK / 64;                       // 9 panels of 64 bf16 (128 bytes)
// Rank r of a pair owns V dims [256r, 256r + 256) = panels 4r .. 4r+3 and contracts S = Q K^T
// over those four panels plus half of panel 8 (dims 512-575, a K-only panel): K steps 2r,
// 2r+1 of its four.  Both ranks issue 18 MMAs per tile.  Each loads five panels of every
// row: its four V panels (local panels 0-3) and panel 8 (local panel 4).
constexpr int kLocalPanels = 5;
constexpr int kKvPanel = N * 128;                      // 8192
constexpr int kStageBytes = kLocalPanels * kKvPanel;   // 40960
// Four stages: at the headline batch a CTA's whole share (four tiles) is in flight at once
constexpr int kStages = 4;
constexpr int kOffKv = 0;
constexpr int kOffX = kOffKv + kStages * kStageBytes;  // the peer's S partial
constexpr int kXBytes = H * N * 4;                     // 32768
constexpr int kXBufs = 1;  // one receive buffer: the sender of tile i waits for the read of i-1
constexpr int kQPanelBytes = H * 128;                  // one 128-head x 64-dim Q panel
constexpr int kOffQ8 = kOffX + kXBufs * kXBytes;       // Q panel 8, the A operand from shared memory
constexpr int kMaxRows = 4096;                         // k <= 4096: a CTA's rows, resolved once
constexpr int kOffRows = kOffQ8 + kQPanelBytes;
constexpr int kOffBar = kOffRows + kMaxRows * 4;
static_assert(kOffQ8 % 1024 == 0, "128-byte swizzled operand needs 1024-byte alignment");
// TMEM columns: O half [0, 256), two S tiles [256, 384) (P of a tile, bf16 pairs, is written
// over the first 32 columns of its own S tile once S has been read), this rank's Q panels
// 4r .. 4r+3 [384, 512).  Two S tiles let S(i+1) run while the softmax works on tile i.
constexpr int kSBufs = 2;
constexpr int kTmemS = DVH, kTmemQ = kTmemS + kSBufs * N;
static_assert(kTmemQ + 4 * 32 == 512, "TMEM budget");
// kv_full[kStages] kv_empty[kStages] s_full[2] s_read[2] s_sent[2] x_full[kXBufs]
// x_free[kXBufs] x_read[kXBufs] p_full[2] p_free o_done q_full q_tma merge_full
constexpr int kNumBars = 2 * kStages + 3 * kSBufs + 3 * kXBufs + kSBufs + 5;
// Split merge inside the cluster (after the tiles, in the free stage ring): the CTA owning
// heads [split * hp, + hp) of its V half receives, from every split s, those heads' rows of
// O (bf16, unnormalised, 512 bytes each) at [s][head][512 B] and their (max, sum) at
// [s][head][16 B]; hp = 128 / nsplit, so both areas are the same size for every split count.
constexpr int kOffMerge = kOffKv;
constexpr int kOffMergeMl = kOffMerge + H * 512;
static_assert(kOffMergeMl + H * 16 <= kStages * kStageBytes, "merge buffers fit the stage ring");
// Q arrives by TMA (one 128-head x 64-dim box per panel, 128-byte swizzle): panels 4r .. 4r+3
// in the KV stage buffers, which the row gathers use only once Q has moved on into TMEM, and
// panel 8 straight into its own buffer
// Q is staged in stages 2-3, so that the gathers of tiles 0 and 1 need not wait for it
constexpr int kOffQStage = 2 * kStageBytes;
static_assert(kOffQStage % 1024 == 0 && kOffQStage + 4 * kQPanelBytes <= kStages * kStageBytes,
              "Q staging fits the KV stages");
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kSmem = 1024 + kOffTmem + 16;
// warps 0-3 softmax and 4-7 S senders (warp w reads TMEM lanes 32(w%4) .. +31),
// warp 8 MMA issue, warp 9 credit forwarding, warps 10-13 row gathers
constexpr int kMmaWarp = 8;
constexpr int kFwdWarp = 9;
constexpr int kLoadWarp0 = 10;
constexpr int kLoadWarps = 4;  // a warp issues its TMA ops one lane at a time: spread them
constexpr int kThreads = (kLoadWarp0 + kLoadWarps) * 32;               // 448
constexpr int kGathers = (N / 4) * kLocalPanels;                        // 80 gather4 per tile
constexpr int kGathersPerWarp = kGathers / kLoadWarps;                  // 20
static_assert(kGathers % kLoadWarps == 0 && kGathersPerWarp <= 32, "gathers per warp");
static_assert(kSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kIdescS = make_idesc(1 /*bf16*/, 128, N, false, false);
constexpr uint32_t kIdescO = make_idesc(1 /*bf16*/, 128, DVH, false, true);
constexpr int kMergeBatch = 8;  // the most splits the in-cluster merge takes (the cluster's 16 CTAs)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Global panel of local panel lp of rank r.
__host__ __device__ constexpr int global_panel(int rank, int lp) { return lp < 4 ? 4 * rank + lp : 8; }
}  // namespace mla

// This rank's four TMEM Q panels (head h's row), staged in shared memory by TMA (128-byte
// swizzle: 16-byte chunk j of row h sits at chunk j ^ (h & 7)), into TMEM lane h as the MMA's
// A operand: 64 dims = 32 columns per panel, two bf16 per column.  Every thread of warps
// 0-3, converged.
__device__ __forceinline__ void load_q_tmem(const uint8_t* q_smem, int h, uint32_t t_row) {
  using namespace mla;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    const uint4* row = (const uint4*)(q_smem + c * kQPanelBytes + h * 128);
    float f[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 v = row[j ^ (h & 7)];
      f[4 * j] = __uint_as_float(v.x);
      f[4 * j + 1] = __uint_as_float(v.y);
      f[4 * j + 2] = __uint_as_float(v.z);
      f[4 * j + 3] = __uint_as_float(v.w);
    }
    tmem_st32(t_row + c * 32, f);
  }
  tmem_wait_st();
}

// One cluster of two CTAs = (request b, KV split); rank r of the pair produces output
// dims [256r, 256r + 256).  Per 64-row tile, each CTA gathers its five 64-dim panels of the
// selected rows (TMA gather4 into a three-stage ring), forms its part of S = Q K^T over its
// latent dims in TMEM (four Q panels in TMEM and Q panel 8 in shared memory are the A
// operands), sends that 128 x 64 partial to the other CTA through distributed shared memory
// and adds the one it receives, so both hold the same S (fp32 addition commutes, so the two
// sums are bit-identical) and run the same online softmax (one thread per head).  S tiles
// alternate between two TMEM buffers, so the MMAs of S(i+1) overlap the exchange and softmax
// of tile i.  P goes back over its own S tile as bf16 pairs (the A operand of PV) and
// O_half += P V_half accumulates in TMEM (256 columns).
__global__ void __launch_bounds__(mla::kThreads, 1)
    attn_mla_tc(const AttnParams p, const __grid_constant__ CUtensorMap kv_map,
                const __grid_constant__ CUtensorMap q_map) {
  using namespace mla;
  extern __shared__ uint8_t sm_raw_a[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)sm_raw_a + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;   // S partial of the tile in TMEM buffer i % 2
  uint64_t* s_read = s_full + kSBufs;      // ... read by the senders and the softmax
  uint64_t* s_sent = s_read + kSBufs;      // ... read by the senders (P may overwrite it)
  uint64_t* x_full = s_sent + kSBufs;      // the other rank's partial has arrived here
  uint64_t* x_free = x_full + kXBufs;      // the other rank has read our partial (credit)
  uint64_t* x_read = x_free + kXBufs;      // our softmax has read receive buffer b
  uint64_t* p_full = x_read + kXBufs;      // P of the tile in buffer i % 2 is in TMEM
  uint64_t* p_free = p_full + kSBufs;      // PV of the latest tile has finished
  uint64_t* o_done = p_free + 1;
  uint64_t* q_full = p_free + 2;
  uint64_t* q_tma = p_free + 3;
  uint64_t* merge_full = p_free + 4;       // every split's rows for this CTA's heads have landed
  uint32_t* tmem_slot = (uint32_t*)(sm + kOffTmem);
  __shared__ int s_abort;
  __shared__ uint64_t s_mask[kStages];  // valid rows of the tile in each stage

  const int b = blockIdx.y;
  const uint32_t crank = cluster_rank();  // == blockIdx.x (the cluster spans the splits)
  const int rank = (int)(crank & 1u);      // which half of V
  const uint32_t peer_crank = crank ^ 1u;  // the other CTA of the pair
  const int split = blockIdx.x >> 1;
  const int warp = warp_id(), lane = lane_id();
  const int T_all = (p.k + N - 1) / N;
  const int t0 = (int)(((long long)T_all * split) / p.nsplit);
  const int t1 = (int)(((long long)T_all * (split + 1)) / p.nsplit);
  const int my_tiles0 = t1 - t0;  // tiles of this CTA's share of the selection
  // with n_valid the share is known only after the kernel before has finished: what runs
  // ahead of that is sized for the most tiles a share can get
  const int my_tiles_max = p.n_valid ? (T_all + p.nsplit - 1) / p.nsplit : my_tiles0;
  const uint32_t sbase = smem_u32(sm);

  // With a ready count the gather warps resolve this CTA's rows (selection -> page table ->
  // shared memory) as soon as this request's selection is complete, before they join the
  // set-up barrier: a CTA that started late (on an SM the kernel before had held) resolves
  // its rows while its other warps set up, instead of after them.
  constexpr int kRStep = kLoadWarps * 32;
  int* s_rows = (int*)(sm + kOffRows);
  auto resolve_rows = [&](int tb_, int ntiles, const int* spec_sv, bool spec_ok) {
    const int lw = warp - kLoadWarp0;
    const int nrows = ntiles * N;
    for (int r0 = lw * 32 + lane; r0 < nrows; r0 += 4 * kRStep) {
      int sv[4];  // four rows' selections, then their page-table lookups, in flight together
      const bool spec = spec_ok && r0 < kRStep;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + u * kRStep, j = tb_ * N + r;
        sv[u] = (r < nrows && j < p.k) ? (spec ? spec_sv[u] : p.sel[(size_t)b * p.k + j]) : -1;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + u * kRStep;
        const long long row = attn_row(p, b, sv[u]);
        if (r < nrows) s_rows[r] = row >= 0 ? (int)row : (int)p.num_rows;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kLoadWarps * 32) : "memory");  // the gather warps only
  };
  const bool early_rows = p.ready != nullptr;  // (then the share is the split's: t0 .. t1)
  if (early_rows && warp >= kLoadWarp0) {
    if (p.addressing == LS_ROWS_PAGED) {
      const int* pt = p.page_table + (size_t)b * p.max_pages;
      for (int i = ((warp - kLoadWarp0) * 32 + lane) * 32; i < p.max_pages; i += kLoadWarps * 32 * 32)
        prefetch_l2(pt + i);
    }
    if (lane == 0) wait_count(p.ready + b, p.ready_want);
    __syncwarp();
    resolve_rows(t0, my_tiles0, nullptr, false);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], kLoadWarps);  // each gather warp arrives with its bytes
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_read[s], 256);  // this CTA's sender and softmax threads
      mbar_init(&s_sent[s], 128);  // this CTA's sender threads
      mbar_init(&p_full[s], 128);  // this CTA's softmax threads
    }
    for (int s = 0; s < kXBufs; ++s) {
      mbar_init(&x_full[s], 1);  // armed with the partial's bytes; the other CTA's stores land on it
      mbar_init(&x_free[s], 1);    // the other CTA's forwarding thread, remotely
      mbar_init(&x_read[s], 128);  // this CTA's softmax threads
    }
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    mbar_init(q_full, 128);  // the softmax threads, once Q is in TMEM (and out of the stages)
    mbar_init(q_tma, 1);
    mbar_init(merge_full, 1);
    // armed now; the rows arrive only after the cluster-wide barrier that follows the tiles
    if (p.merge) mbar_arrive_expect_tx(merge_full, (uint32_t)(H * (512 + 16)));
    s_abort = 0;
    fence_mbar_init();
    // Q is an input of the step, never written by the kernel before: fetch it at once
    if (my_tiles_max > 0) {
      mbar_arrive_expect_tx(q_tma, 5 * kQPanelBytes);
      for (int c = 0; c < 4; ++c)
        tma_load_2d(sbase + kOffQStage + c * kQPanelBytes, &q_map, q_tma, global_panel(rank, c) * 64, b * H);
      tma_load_2d(sbase + kOffQ8, &q_map, q_tma, 8 * 64, b * H);
    }
    // arm the receive buffers for the first tiles before the other CTA can send (an armed
    // buffer that no tile uses is never waited on)
    for (int s = 0; s < kXBufs && s < my_tiles_max; ++s) mbar_arrive_expect_tx(&x_full[s], kXBytes);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  // the other CTA may address this one's barriers and receive buffers once it has seen
  // this arrival; only the warps that write to the other CTA wait for it early (the rest
  // wait before the final barrier), so the row gathers need not
  cluster_arrive();
  bool cluster_waited = false;
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem;          // columns [0, 256): O half
  const uint32_t tm_s = tmem + kTmemS;  // two S tiles (P over the first half of each)
  const uint32_t tm_q = tmem + kTmemQ;  // this rank's Q panels 4r .. 4r+3
  if (warp < 4 && my_tiles_max > 0) {
    // a wait that gives up (recorded in the device status) aborts the whole CTA
    if (mbar_wait(q_tma, 0)) {
      load_q_tmem(sm + kOffQStage, threadIdx.x, tm_q + ((uint32_t)(warp * 32) << 16));
      tc_fence_before();
    } else if (threadIdx.x == 0) {
      s_abort = 1;
    }
    mbar_arrive(q_full);
  }
  if (warp >= kLoadWarp0 && p.addressing == LS_ROWS_PAGED && !early_rows) {
    // the page table is an input of the step: warm its rows for this request in L2
    const int* pt = p.page_table + (size_t)b * p.max_pages;
    for (int i = ((warp - kLoadWarp0) * 32 + lane) * 32; i < p.max_pages; i += kLoadWarps * 32 * 32)
      prefetch_l2(pt + i);
  }
  // under programmatic dependent launch everything above overlaps the kernel before;
  // the selection, the rows and the outputs are touched only after it has finished.  With a
  // ready count only the gather warps read what the kernel before wrote (the selection), so
  // only they wait, for this request's part of it: the other warps go on (a CTA that started
  // late finishes its prologue meanwhile) and size their work from the split alone
  if (!p.ready) griddep_wait();
  griddep_launch_dependents();
  // the gather warps load the selections of their first rows (for the usual tile range)
  // while the tile range is settled below, so that the two loads overlap
  int spec_sv[4];
  if (warp >= kLoadWarp0 && !early_rows) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = (warp - kLoadWarp0) * 32 + lane + u * kRStep, j = t0 * N + r;
      spec_sv[u] = (r < my_tiles0 * N && j < p.k) ? p.sel[(size_t)b * p.k + j] : -1;
    }
  }
  // in a compacted selection a share that starts with padding holds no row at all (the
  // tail of a miss list): such a CTA only writes an empty partial
  int tb = t0, my_tiles = my_tiles0;
  if (p.n_valid) {
    const int nv = min(max(p.n_valid[b], 0), p.k);
    const int tv = (nv + N - 1) / N;
    tb = (int)(((long long)tv * split) / p.nsplit);
    my_tiles = min((int)(((long long)tv * (split + 1)) / p.nsplit) - tb, my_tiles_max);
  } else if (p.compacted && !p.ready && my_tiles0 > 0 && p.sel[(size_t)b * p.k + (size_t)t0 * N] < 0) {
    my_tiles = 0;  // (with a ready count a share of padding is gathered as zero rows and masked)
  }
  const size_t pslot = (size_t)b * p.nsplit_total + p.split_base + split;  // partial slot
  // the softmax threads' final running max and sum, and whether O in TMEM is complete
  // (for the split merge after the cluster-wide barrier)
  float m_out = -INFINITY, l_out = 0.f;
  bool o_ready = false;

  if (warp >= kLoadWarp0) {
    // ================= row gathers: tile i goes to stage i % kStages =================
    // The gather warps first resolve all of this CTA's rows (selection -> page table) into
    // shared memory.  A tile's 16 groups of 4 rows x 5 panels are then 80 TMA gather4
    // loads; gather e (group e % 16, local panel e / 16) is issued by lane e % 20 of gather
    // warp e / 20, each landing as four 128-byte-swizzled lines of its panel.  Padding rows
    // point one past the pool, which the TMA unit fills with zeros; the softmax masks them.
    const int lw = warp - kLoadWarp0;
    const int e = lw * kGathersPerWarp + lane;  // this lane's gather (if lane < 20)
    const int lx = e % (N / 4), lp = e / (N / 4);
    // resolve all of this CTA's rows once (out-of-range marker: one past the pool), unless
    // that was done ahead of the set-up
    if (!early_rows) resolve_rows(tb, my_tiles, spec_sv, tb == t0 && my_tiles <= my_tiles0);
    for (int i = 0; i < my_tiles; ++i) {
      const int st = i % kStages;
      int go = 1;
      if (lane == 0) {  // one lane decides, so the warp stays converged
        // the first tiles of stages 2 and 3 land where Q was staged: only once Q is in TMEM
        go = i >= kStages ? mbar_wait(&kv_empty[st], ((i / kStages) - 1) & 1) : (i < 2 || mbar_wait(q_full, 0));
        if (*(volatile int*)&s_abort) go = 0;
        if (!go) s_abort = 1;
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) break;
      uint64_t vmask = 0;
#pragma unroll
      for (int h32 = 0; h32 < N / 32; ++h32)
        vmask |= (uint64_t)__ballot_sync(0xffffffffu, s_rows[i * N + h32 * 32 + lane] < (int)p.num_rows) << (32 * h32);
      if (lane == 0) {
        if (lw == 0) s_mask[st] = vmask;
        mbar_arrive_expect_tx(&kv_full[st], kGathersPerWarp * 512);
      }
      __syncwarp();
      if (lane < kGathersPerWarp) {
        const int* rr = s_rows + i * N + 4 * lx;
        tma_gather4(sbase + kOffKv + st * kStageBytes + lp * kKvPanel + lx * 512, &kv_map, &kv_full[st],
                    global_panel(rank, lp) * 64, rr[0], rr[1], rr[2], rr[3]);
      }
    }
    // never leave with copies in flight (the tiles of the last kStages loads)
    if (lane == 0)
      for (int i = max(0, my_tiles - kStages); i < my_tiles; ++i) mbar_wait(&kv_full[i % kStages], (i / kStages) & 1);
    __syncwarp();
  } else if (warp == kFwdWarp) {
    // ================= credit forwarding =================
    // Once this CTA's softmax has read receive buffer b (tile j), re-arm its barrier for
    // tile j + kXBufs and tell the other CTA's senders they may write it.  The remote
    // arrival (a cluster-scope release) is slow, so it is kept off the softmax warps.
    cluster_wait();
    cluster_waited = true;
    if (lane == 0) {
      const uint32_t xfree_peer = dsmem_map(smem_u32(x_free), peer_crank);
      for (int j = 0; j + kXBufs < my_tiles; ++j) {
        const int xb = j % kXBufs;
        if (!mbar_wait(&x_read[xb], (j / kXBufs) & 1)) break;
        mbar_arrive_expect_tx(&x_full[xb], kXBytes);
        mbar_arrive_remote(xfree_peer + xb * 8);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer: event driven =================
    // S(i) goes out whole once tile i has landed and S buffer i % 2 is free again: tile
    // i-2's S has been read (by the senders and the softmax) and PV(i-2), which reads P(i-2)
    // from the same columns, has been issued (the tensor pipe runs one thread's MMAs in
    // order).  PV(i) goes out as soon as P(i) is ready.  Neither blocks the other.
    if (lane == 0 && my_tiles > 0) {
      const uint32_t q8 = sbase + kOffQ8;
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      int ns = 0, npv = 0;
      uint64_t idle_since = 0;
      while (ok && npv < my_tiles) {
        bool progressed = false;
        if (npv < ns && mbar_test_wait(&p_full[npv % kSBufs], (npv / kSBufs) & 1)) {
          tc_fence_after();
          // this rank's V half is local panels 0-3 of the stage; P(npv) sits over its S tile
          const uint32_t v = sbase + kOffKv + (npv % kStages) * kStageBytes;
          const uint32_t pa = tm_s + (npv % kSBufs) * N;
#pragma unroll
          for (int kk = 0; kk < N / 16; ++kk) {
            const uint64_t bd = make_sdesc(v + kk * 16 * 128, kKvPanel, 1024, kSwizzle128);
            mma_bf16_ta(tm_o, pa + kk * 8, bd, kIdescO, (npv > 0 || kk > 0));
          }
          tc_commit(&kv_empty[npv % kStages]);
          tc_commit(p_free);
          ++npv;
          progressed = true;
        }
        // S(i): 16 K steps over the TMEM Q panels, then this rank's two steps of panel 8
        // with Q from shared memory.  Each MMA waits on the previous one (same
        // accumulator), so S costs about as many MMA latencies as it has K steps.
        if (ns < my_tiles &&
            (ns < kSBufs || (npv >= ns - 1 && mbar_test_wait(&s_read[ns % kSBufs], ((ns / kSBufs) - 1) & 1))) &&
            mbar_test_wait(&kv_full[ns % kStages], (ns / kStages) & 1)) {
          tc_fence_after();
          const uint32_t kv = sbase + kOffKv + (ns % kStages) * kStageBytes;
          const uint32_t sb = tm_s + (ns % kSBufs) * N;
#pragma unroll 1
          for (int pn = 0; pn < 4; ++pn) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = make_sdesc(kv + pn * kKvPanel + kk * 32, 16, 1024, kSwizzle128);
              mma_bf16_ta(sb, tm_q + pn * 32 + kk * 8, bd, kIdescS, (pn | kk) != 0);
            }
          }
#pragma unroll
          for (int kk = 2 * rank; kk < 2 * rank + 2; ++kk) {
            const uint64_t ad = make_sdesc(q8 + kk * 32, 16, 1024, kSwizzle128);
            const uint64_t bd = make_sdesc(kv + 4 * kKvPanel + kk * 32, 16, 1024, kSwizzle128);
            mma_bf16(sb, ad, bd, kIdescS, 1);
          }
          tc_commit(&s_full[ns % kSBufs]);
          ++ns;
          progressed = true;
        }
        if (progressed) {
          idle_since = 0;
        } else {
          // nothing to issue yet: step aside briefly, so that this polling loop does not take
          // issue slots from the softmax warp that shares its scheduler
          __nanosleep(64);
          const uint64_t now = globaltimer();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > *(volatile unsigned long long*)&g_wait_limit_ns) {
            flag(LS_DEV_TIMEOUT);
            ok = false;
          }
        }
      }
      if (!ok) s_abort = 1;
      tc_commit(o_done);
    }
  } else if (warp >= 4) {
    // ================= S senders: warps 4..7, thread = head =================
    // This rank's partial S of each tile goes from TMEM to the other CTA as asynchronous
    // stores that count their bytes on the receiver's barrier (armed by the receiver for
    // each tile).  The other CTA's receive buffer is written for tile i only after that CTA's
    // softmax has read tile i - kXBufs from it and its forwarding thread has re-armed the
    // barrier (x_free credit), so the senders run ahead of both softmaxes by kXBufs tiles.
    const int q = warp & 3;
    const int h = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t peer = peer_crank;
    // partials are stored chunk-major (chunk c of head h at c * 2048 + h * 16), so a
    // warp's 16-byte accesses are consecutive
    const uint32_t x_peer = dsmem_map(sbase + kOffX, peer);
    const uint32_t xfull_peer = dsmem_map(smem_u32(x_full), peer);
    cluster_wait();
    cluster_waited = true;
    for (int i = 0; i < my_tiles; ++i) {
      const int sb = i % kSBufs, xb = i % kXBufs;
      // every wait in front of a warp-collective TMEM access is decided for the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (i / kSBufs) & 1))) break;
      tc_fence_after();
      float cur[N];
      tmem_ld64(tm_s + lane_off + sb * N, cur);
      tc_fence_before();
      mbar_arrive(&s_read[sb]);
      mbar_arrive(&s_sent[sb]);  // the softmax may now write P over this S tile
      if (i >= kXBufs && !__all_sync(0xffffffffu, mbar_wait_cluster(&x_free[xb], ((i / kXBufs) - 1) & 1))) break;
#pragma unroll
      for (int c = 0; c < N / 4; ++c)
        st_async_v4(x_peer + xb * kXBytes + c * 2048 + h * 16, cur[4 * c], cur[4 * c + 1], cur[4 * c + 2],
                    cur[4 * c + 3], xfull_peer + xb * 8);
    }
  } else {
    // ================= softmax: warps 0..3, thread = head =================
    const int h = warp * 32 + lane;
    const float sl2 = p.scale * kLog2e;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < my_tiles; ++i) {
      const int st = i % kStages, sb = i % kSBufs, xb = i % kXBufs;
      // the loaders published the tile's valid rows with their kv_full arrivals
      if (!__all_sync(0xffffffffu, mbar_wait(&kv_full[st], (i / kStages) & 1))) { ok = false; break; }
      const uint64_t vmask = s_mask[st];
      // S = this rank's partial (TMEM) + the other rank's (receive buffer xb)
      // every wait in front of a warp-collective TMEM access is decided for the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (i / kSBufs) & 1))) { ok = false; break; }
      tc_fence_after();
      float s[N];
      tmem_ld64(tm_s + lane_off + sb * N, s);
      tc_fence_before();
      mbar_arrive(&s_read[sb]);  // with the senders' reads, this frees the S buffer
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(&x_full[xb], (i / kXBufs) & 1))) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < N / 4; ++c) {
        const float4 o = *(const float4*)(sm + kOffX + xb * kXBytes + c * 2048 + h * 16);
        s[4 * c] += o.x;
        s[4 * c + 1] += o.y;
        s[4 * c + 2] += o.z;
        s[4 * c + 3] += o.w;
      }
      mbar_arrive(&x_read[xb]);  // the forwarding thread re-arms buffer xb and passes the credit
      // a tile whose rows are all valid (every tile but a ragged last one) skips the masking;
      // max and sum run as four independent chains
      const bool full = vmask == ~0ull;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int r = 0; r < N; ++r) m4[r & 3] = fmaxf(m4[r & 3], s[r]);
      } else {
#pragma unroll
        for (int r = 0; r < N; ++r)
          if ((vmask >> r) & 1u) m4[r & 3] = fmaxf(m4[r & 3], s[r]);
      }
      const float tmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mt = tmax * sl2;
      float factor = 1.f;
      bool rescale = false;
      if (mt > m_run + 8.f) {  // also true for the first tile with data
        if (m_run != -INFINITY) {
          factor = exp2f(m_run - mt);
          rescale = true;
        }
        m_run = mt;
      }
      float p4[4] = {0.f, 0.f, 0.f, 0.f};  // s becomes P in place
      if (full) {
#pragma unroll
        for (int r = 0; r < N; ++r) {
          s[r] = ex2_ftz(fmaf(s[r], sl2, -m_run));
          p4[r & 3] += s[r];
        }
      } else {
#pragma unroll
        for (int r = 0; r < N; ++r) {
          s[r] = ((vmask >> r) & 1u) ? ex2_ftz(fmaf(s[r], sl2, -m_run)) : 0.f;
          p4[r & 3] += s[r];
        }
      }
      const float psum = (p4[0] + p4[1]) + (p4[2] + p4[3]);
      // tcgen05.ld/st are warp-collective: the whole warp rescales when any lane must
      // (lanes that need not have factor 1).  O may be rescaled only once PV(i-1) has
      // finished adding into it (a rescale never happens at the first tile).
      if (__any_sync(0xffffffffu, rescale)) {
        if (!__all_sync(0xffffffffu, mbar_wait(p_free, (i - 1) & 1))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < DVH; c0 += 32) {
          float v[32];
          tmem_ld32(tm_o + lane_off + c0, v);
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] *= factor;
          tmem_st32(tm_o + lane_off + c0, v);
        }
        tmem_wait_st();
      }
      l_run = l_run * factor + psum;
      // P(i) into TMEM lane h over the first 32 columns of its own S tile: column c holds
      // rows 2c, 2c+1 as bf16 -- once the senders have read that S tile
      float pw[N / 2];
#pragma unroll
      for (int c = 0; c < N / 2; ++c) {
        __nv_bfloat162 two = __floats2bfloat162_rn(s[2 * c], s[2 * c + 1]);
        pw[c] = __uint_as_float(*(uint32_t*)&two);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&s_sent[sb], (i / kSBufs) & 1))) { ok = false; break; }
      tc_fence_after();
      tmem_st32(tm_s + lane_off + sb * N, pw);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    // ---- epilogue
    bool fin = ok && my_tiles > 0 && mbar_wait(o_done, 0);
    fin = __all_sync(0xffffffffu, fin);  // the TMEM reads below are warp-collective
    m_out = m_run;
    l_out = l_run;
    o_ready = fin;
    if (p.merge) {
      // the splits are merged after the cluster-wide barrier below
    } else if (fin) {
      tc_fence_after();
      const bool single = p.nsplit_total == 1;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // 64 columns per TMEM load (half the round trips), stored 32 at a time
      for (int c64 = 0; c64 < DVH; c64 += 64) {
        float v64[64];
        tmem_ld64(tm_o + lane_off + c64, v64);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int c0 = c64 + 32 * hh;
          const float* v = v64 + 32 * hh;
          if (single && p.o_f32) {
            float4* o = (float4*)((float*)p.o + ((size_t)b * H + h) * DV + rank * DVH + c0);
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              o[c / 4] = make_float4(v[c] * inv, v[c + 1] * inv, v[c + 2] * inv, v[c + 3] * inv);
          } else if (single) {
            __nv_bfloat16* o = (__nv_bfloat16*)p.o + ((size_t)b * H + h) * DV + rank * DVH + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 two = __floats2bfloat162_rn(v[c + 2 * e] * inv, v[c + 2 * e + 1] * inv);
                w[e] = *(uint32_t*)&two;
              }
              *(uint4*)(o + c) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else if (p.o_f32) {
            // float32 partials, layout [b][split][dim / 4][head][4]: a warp's store is 512
            // contiguous bytes
            float4* o = (float4*)p.part_o + (pslot * (DV / 4) + (rank * DVH + c0) / 4) * H + h;
            const bool any = l_run > 0.f;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              o[(size_t)(c / 4) * H] = any ? make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            // for a bf16 output the partials are bf16 too (one more rounding of what is rounded
            // to bf16 at the end), layout [b][split][dim / 8][head][8]: a warp's store is 512
            // contiguous bytes
            uint4* o = (uint4*)p.part_o + (pslot * (DV / 8) + (rank * DVH + c0) / 8) * H + h;
            const float any = l_run > 0.f ? 1.f : 0.f;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 two = __floats2bfloat162_rn(v[c + 2 * e] * any, v[c + 2 * e + 1] * any);
                w[e] = *(uint32_t*)&two;
              }
              o[(size_t)(c / 8) * H] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      if (rank == 0) {  // both ranks hold the same running max and sum
        if (single) {
          p.lse[(size_t)b * H + h] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        } else {
          float* ml = p.part_ml + (pslot * H + h) * 2;
          ml[0] = l_run > 0.f ? m_run : -INFINITY;
          ml[1] = l_run;
        }
      }
    } else if (my_tiles == 0 && p.nsplit_total > 1) {
      if (p.o_f32) {
        float4* o = (float4*)p.part_o + (pslot * (DV / 4) + rank * DVH / 4) * H + h;
        for (int c = 0; c < DVH / 4; ++c) o[(size_t)c * H] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        uint4* o = (uint4*)p.part_o + (pslot * (DV / 8) + rank * DVH / 8) * H + h;
        for (int c = 0; c < DVH / 8; ++c) o[(size_t)c * H] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (rank == 0) {
        float* ml = p.part_ml + (pslot * H + h) * 2;
        ml[0] = -INFINITY;
        ml[1] = 0.f;
      }
    }
    if (p.done && !p.merge) {
      // this CTA's part of the split partial is stored (every path above ends here):
      // count it for the combine
      asm volatile("bar.sync 2, 128;" ::: "memory");  // the four softmax warps
      count_done(p.done + b);
    }
  }
  // every warp must reach the barrier converged (the MMA warp's lane 0 arrives last).
  // The cluster-wide barrier also keeps this CTA's shared memory alive until the other
  // CTAs have made their last remote writes and arrivals; only then may TMEM be released.
  __syncwarp();
  if (!cluster_waited) cluster_wait();
  if (p.merge) {
    // ================= split merge inside the cluster =================
    // Past this barrier every CTA of the request has finished its tiles: its stage ring is
    // free and every remote store into it has landed.
    tc_fence_before();
    cluster_sync_all();
    const int hp = H / p.nsplit;
    if (warp < 4) {
      // thread = head h: its unnormalised O row over this CTA's V half (bf16, like a split
      // partial) and its (max, sum) go to the CTA of this rank that owns head h
      tc_fence_after();
      const int h = threadIdx.x;
      const int owner = h / hp, hl = h - owner * hp;
      const uint32_t dst = (uint32_t)(2 * owner + rank);
      const uint32_t bar_dst = dsmem_map(smem_u32(merge_full), dst);
      const uint32_t row_dst = dsmem_map(sbase + kOffMerge + (uint32_t)((split * hp + hl) * 512), dst);
      const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
      const float any = (o_ready && l_out > 0.f) ? 1.f : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < DVH; c0 += 32) {
        float v[32];
        if (o_ready) {
          tmem_ld32(tm_o + lane_off + c0, v);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 two = __floats2bfloat162_rn(v[c + 2 * e] * any, v[c + 2 * e + 1] * any);
            w[e] = *(uint32_t*)&two;
          }
          st_async_v4_b32(row_dst + (uint32_t)(c0 + c) * 2, w[0], w[1], w[2], w[3], bar_dst);
        }
      }
      const float m_send = any > 0.f ? m_out : -INFINITY, l_send = any > 0.f ? l_out : 0.f;
      st_async_v4(dsmem_map(sbase + kOffMergeMl + (uint32_t)((split * hp + hl) * 16), dst), m_send, l_send, 0.f,
                  0.f, bar_dst);
    }
    if (warp < 8) {
      // heads [split * hp, + hp) x this rank's 256 dims, 8 dims per item: the same weights and
      // summation order as attn_combine, so both ways give the same bits
      const bool got = __all_sync(0xffffffffu, mbar_wait(merge_full, 0));
      const int ns = p.nsplit;
      for (int item = threadIdx.x; got && item < hp * 32; item += 256) {
        const int hl = item >> 5, j = item & 31, h = split * hp + hl;
        float mv[kMergeBatch], lv[kMergeBatch], x[kMergeBatch][8];
#pragma unroll
        for (int s2 = 0; s2 < kMergeBatch; ++s2) {
          const int sc = min(s2, ns - 1);
          const float4 ml4 = *(const float4*)(sm + kOffMergeMl + (sc * hp + hl) * 16);
          mv[s2] = ml4.x;
          lv[s2] = ml4.y;
          const uint4 u = *(const uint4*)(sm + kOffMerge + (sc * hp + hl) * 512 + j * 16);
          const uint32_t q4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*(const __nv_bfloat162*)&q4[e]);
            x[s2][2 * e] = f.x;
            x[s2][2 * e + 1] = f.y;
          }
        }
        float M = -INFINITY, Lsum = 0.f, acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kMergeBatch; ++s2) M = fmaxf(M, mv[s2]);
        if (M != -INFINITY) {
#pragma unroll
          for (int s2 = 0; s2 < kMergeBatch; ++s2) {
            const float wgt = (s2 < ns && lv[s2] > 0.f) ? exp2f(mv[s2] - M) : 0.f;
            Lsum += wgt * lv[s2];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, x[s2][e], acc[e]);
          }
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        uint32_t wo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __nv_bfloat162 two = __floats2bfloat162_rn(acc[2 * q] * inv, acc[2 * q + 1] * inv);
          wo[q] = *(uint32_t*)&two;
        }
        *(uint4*)((__nv_bfloat16*)p.o + ((size_t)b * H + h) * DV + rank * DVH + j * 8) =
            make_uint4(wo[0], wo[1], wo[2], wo[3]);
        if (rank == 0 && j == 0) p.lse[(size_t)b * H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge split-KV partials: o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One thread per (request, head, 8 consecutive dims); grid (H * DV / 8 / 256, B), 256
// threads.  A warp covers 32 consecutive heads at the same dims, so each of its partial
// reads is a 512-byte run of the [dim / 4][head][4] (float32) or [dim / 8][head][8] (bf16)
// layout; the 16-byte loads of a thread (2 or 1 per split) are independent of one another.
constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 8;  // splits whose loads are in flight together

// One split's 8 dims of the partial, as float.
template <bool F32>
__device__ __forceinline__ void load_part8(const AttnParams& p, int b, int s, int h, int d0, float* x) {
  using namespace mla;
  if constexpr (F32) {
    const float4* po = (const float4*)p.part_o + (((size_t)b * p.nsplit_total + s) * (DV / 4) + d0 / 4) * H + h;
    const float4 u = po[0], w = po[H];
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
  } else {
    const uint4 u = *((const uint4*)p.part_o + (((size_t)b * p.nsplit_total + s) * (DV / 8) + d0 / 8) * H + h);
    const uint32_t q4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*(const __nv_bfloat162*)&q4[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  }
}

// The weighted sum over the splits, kCombineBatch splits at a time.  Every load of a batch
// (max, sum and partial of each split) is issued unconditionally -- slots past the last
// split re-read the last one and get weight 0 -- so that they are all in flight at once.
template <bool F32>
__device__ __forceinline__ void combine_splits(const AttnParams& p, int b, int h, int d0, const float* ml, float M,
                                               float* acc, float& Lsum) {
  const int ns = p.nsplit_total;
  for (int s0 = 0; s0 < ns; s0 += kCombineBatch) {
    float mv[kCombineBatch], lv[kCombineBatch], x[kCombineBatch][8];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      const int s = min(s0 + j, ns - 1);
      mv[j] = ml[(size_t)s * mla::H * 2];
      lv[j] = ml[(size_t)s * mla::H * 2 + 1];
      load_part8<F32>(p, b, s, h, d0, x[j]);
    }
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      // an empty split, or a slot past the last split, adds nothing
      const float wgt = (s0 + j < ns && lv[j] > 0.f) ? exp2f(mv[j] - M) : 0.f;
      Lsum += wgt * lv[j];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, x[j][e], acc[e]);
    }
  }
}

// More splits than one batch holds: the maximum first, then the weighted sum batch by batch.
__device__ __forceinline__ void combine_general(const AttnParams& p, int b, int h, int d0, const float* ml, float& M,
                                                float* acc, float& Lsum) {
  using namespace mla;
  for (int s0 = 0; s0 < p.nsplit_total; s0 += kCombineBatch) {
    float mv[kCombineBatch];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) mv[j] = ml[(size_t)min(s0 + j, p.nsplit_total - 1) * H * 2];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) M = fmaxf(M, mv[j]);
  }
  if (M != -INFINITY) {
    if (p.o_f32) {
      combine_splits<true>(p, b, h, d0, ml, M, acc, Lsum);
    } else {
      combine_splits<false>(p, b, h, d0, ml, M, acc, Lsum);
    }
  }
}

__global__ void __launch_bounds__(kCombineThreads) attn_combine(const AttnParams p) {
  using namespace mla;
  const int b = blockIdx.y;
  if (p.done) {
    // the partials of request b are complete once all 2 * nsplit of its attention CTAs have
    // counted themselves (this kernel runs only after every one of them has started, so the
    // wait cannot hold a slot one of them needs); one thread polls, the rest wait at the barrier
    if (threadIdx.x == 0) wait_count(p.done + b, 2 * p.nsplit_total);
    __syncthreads();
  } else {
    griddep_wait();  // the partials come from the kernel before
  }
  const int item = blockIdx.x * kCombineThreads + threadIdx.x;
  const int g = item / H, h = item - g * H, d0 = g * 8;
  const float* ml = p.part_ml + (size_t)b * p.nsplit_total * H * 2 + (size_t)h * 2;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float Lsum = 0.f, M = -INFINITY;
  if (p.nsplit_total <= kCombineBatch) {
    // every split in one batch: the maxima, sums and partials of all splits are loaded
    // together (one round trip), then weighted and summed in split order
    const int ns = p.nsplit_total;
    float mv[kCombineBatch], lv[kCombineBatch], x[kCombineBatch][8];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      const int s = min(j, ns - 1);
      mv[j] = ml[(size_t)s * H * 2];
      lv[j] = ml[(size_t)s * H * 2 + 1];
      if (p.o_f32) {
        load_part8<true>(p, b, s, h, d0, x[j]);
      } else {
        load_part8<false>(p, b, s, h, d0, x[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) M = fmaxf(M, mv[j]);
    if (M != -INFINITY) {
#pragma unroll
      for (int j = 0; j < kCombineBatch; ++j) {
        const float wgt = (j < ns && lv[j] > 0.f) ? exp2f(mv[j] - M) : 0.f;
        Lsum += wgt * lv[j];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, x[j][e], acc[e]);
      }
    }
  } else {
    combine_general(p, b, h, d0, ml, M, acc, Lsum);
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  if (p.o_f32) {
    float4* o = (float4*)((float*)p.o + ((size_t)b * H + h) * DV + d0);
    o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 two = __floats2bfloat162_rn(acc[2 * q] * inv, acc[2 * q + 1] * inv);
      w[q] = *(uint32_t*)&two;
    }
    *(uint4*)((__nv_bfloat16*)p.o + ((size_t)b * H + h) * DV + d0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (d0 == 0) p.lse[(size_t)b * H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
}

// Merge of normalised partial attention outputs over disjoint row sets (the shards of a
// context-parallel request): LSE = ln sum_g exp(lse_g), o = sum_g exp(lse_g - LSE) o_g.
// One thread per (request, head, 4 dims).
struct MergeParams {
  int G, B, H, DV, o_f32;
  const float* o_parts;    // [G,B,H,DV]
  const float* lse_parts;  // [G,B,H]
  void* o;                 // [B,H,DV]
  float* lse;              // [B,H]
};

__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeParams p) {
  const long long item = (long long)blockIdx.x * 256 + threadIdx.x;
  const int per_head = p.DV / 4;
  if (item >= (long long)p.B * p.H * per_head) return;
  const int d0 = (int)(item % per_head) * 4;
  const long long bh = item / per_head;  // b * H + h
  const size_t bhs = (size_t)p.B * p.H;
  float M = -INFINITY;
  for (int g = 0; g < p.G; ++g) M = fmaxf(M, p.lse_parts[g * bhs + bh]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
    for (int g = 0; g < p.G; ++g) {
      const float l = p.lse_parts[g * bhs + bh];
      if (l == -INFINITY) continue;
      const float wgt = expf(l - M);
      den += wgt;
      const float4 x = *(const float4*)(p.o_parts + (g * bhs + bh) * p.DV + d0);
      acc.x = fmaf(wgt, x.x, acc.x); acc.y = fmaf(wgt, x.y, acc.y);
      acc.z = fmaf(wgt, x.z, acc.z); acc.w = fmaf(wgt, x.w, acc.w);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  if (p.o_f32) {
    *(float4*)((float*)p.o + bh * p.DV + d0) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    __nv_bfloat162 a2 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    *(uint2*)((__nv_bfloat16*)p.o + bh * p.DV + d0) = make_uint2(*(uint32_t*)&a2, *(uint32_t*)&b2);
  }
  if (d0 == 0) p.lse[bh] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace ls
