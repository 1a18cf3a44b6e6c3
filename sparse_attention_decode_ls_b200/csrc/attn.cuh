// a6. Sparse attention over the selected rows only (LeanSparse, abstract: sparse
// attention limits the history read by each query).
//
//   s_j = scale * q_h . K_j,  o_h = sum_j softmax(s)_j V_j,  lse_h = log sum_j exp(s_j)
//
// * attn_mla_tc: MLA-absorbed decode, 128 query heads against one 576-wide latent KV
//   head whose first 512 dims are V, bf16, on tcgen05 tensor cores.
//     - Heads are the MMA M dimension (128); a tile of 32 selected rows is N.
//     - S = Q K^T (K = 576) and O += P V are tcgen05.mma kind::f16 with f32 TMEM
//       accumulators.  O for all 512 V dims would fill the whole 512-column TMEM,
//       so each CTA owns one 256-wide half of V (the pair recomputes S) and keeps
//       O_half (256 columns) + a double-buffered S (2 x 32 columns) in TMEM.
//     - Rows are gathered through the page table or the hot-buffer slots by TMA: one
//       128-byte box per (row, 64-dim panel), landing swizzled in the row's line of
//       the panel; the same panels serve as the K-major B operand of S and the
//       MN-major B operand of PV.
//     - Online softmax in the exp2 domain with lazy rescaling (O is only rescaled
//       when the running max grows by more than 2^8).
//     - Split-KV across CTAs (enough CTAs to fill the GPU at small batch), merged
//       by attn_combine with the log-sum-exp rule.
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
  int early_q;       // tensor-core kernel: load Q before waiting for the kernel before
};

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
  for (int j = warp; j < p.k; j += 8) {
    const long long r = rows[j];
    float acc = 0.f;
    if (r >= 0) {
      const T* kr = K + r * p.row_stride;
      for (int d = lane; d < p.dk; d += 32) acc = fmaf(qs[d], (float)kr[d], acc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s[j] = r >= 0 ? acc * p.scale : -INFINITY;
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
  for (int d = tid; d < p.dv; d += 256) {
    float acc = 0.f;
    for (int j = 0; j < p.k; ++j) {
      const long long r = rows[j];
      if (r >= 0) acc = fmaf(s[j], (float)V[r * p.row_stride + d], acc);
    }
    o[d] = (T)(l > 0.f ? acc / l : 0.f);
  }
  if (tid == 0) p.lse[(size_t)b * p.H + h] = l > 0.f ? mx + logf(l) : -INFINITY;
}

// =====================================================================================
// tcgen05 MLA kernel
// =====================================================================================
namespace mla {
constexpr int H = 128, DK = 576, DV = 512, DVH = 256, N = 32;
constexpr int kPanels = DK / 64;                       // 9 panels of 64 bf16 (128 bytes)
// The two CTAs of a pair split the latent dims of S = Q K^T: rank 0 takes panels 0-4,
// rank 1 panels 5-8.  Each loads panels 4r .. 4r+4 of every row (its S panels plus its
// half of V: panels 0-3 or 4-7).
constexpr int kLocalPanels = 5;
__host__ __device__ constexpr int s_panels(int rank) { return rank == 0 ? 5 : 4; }  // S panels per rank
constexpr int kQBytes = 5 * H * 128;                   // 81920 (rank 1 uses 65536)
constexpr int kKvPanel = N * 128;                      // 4096
constexpr int kStageBytes = kLocalPanels * kKvPanel;   // 20480
constexpr int kStages = 4;
constexpr int kOffKv = kQBytes;
constexpr int kOffP = kOffKv + kStages * kStageBytes;  // 163840
constexpr int kPBytes = H * N * 2;                     // 8192
constexpr int kOffX = kOffP + kPBytes;                 // 172032: the peer's S partials
constexpr int kXBytes = H * N * 4;                     // 16384 per buffer, two buffers
constexpr int kOffBar = kOffX + 2 * kXBytes;           // 204800
// kv_full[kStages] kv_empty[kStages] s_full[2] x_full[2] sx_full[2] p_full p_free o_done q_full
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 4;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kSmem = 1024 + kOffTmem + 16;
// warps 0-3 softmax and 4-7 S exchange (warp w reads TMEM lanes 32(w%4) .. +31),
// warp 8 MMA issue, warps 9.. loaders: kLoadWarps per KV stage
constexpr int kMmaWarp = 8;
constexpr int kLoadWarps = 2;
constexpr int kThreads = (kMmaWarp + 1 + kStages * kLoadWarps) * 32;    // 544
constexpr int kChunksPerRow = kLocalPanels * 8;                         // 40 16-byte chunks
constexpr int kChunksPerThread = N * kChunksPerRow / (kLoadWarps * 32);  // 20
static_assert(N * kChunksPerRow % (kLoadWarps * 32) == 0, "chunks must split evenly");
static_assert(kSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kIdescS = make_idesc(1 /*bf16*/, 128, N, false, false);
constexpr uint32_t kIdescO = make_idesc(1 /*bf16*/, 128, DVH, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
}  // namespace mla

// This rank's Q panels of request b as 128-row TMA boxes (one 128-byte-swizzled K-major
// panel each).  One thread.
__device__ __forceinline__ void issue_q_load(uint32_t q_smem, const CUtensorMap* q_map, uint64_t* bar, int b,
                                             int rank) {
  using namespace mla;
  const int np = s_panels(rank), p0 = rank * s_panels(0);
  mbar_arrive_expect_tx(bar, (uint32_t)np * H * 128);
#pragma unroll 1
  for (int i = 0; i < np; ++i) tma_load_2d(q_smem + i * (H * 128), q_map, bar, (p0 + i) * 64, b * H);
}

// One cluster of two CTAs = (request b, KV split); rank r of the pair produces output
// dims [256r, 256r + 256).  Per 32-row tile, each CTA gathers its five 64-dim panels of
// the selected rows (cp.async, four stages), forms its part of S = Q K^T over its latent
// dims in TMEM, sends that 128 x 32 partial to the other CTA through distributed shared
// memory and adds the one it receives, so both hold the same S (fp32 addition commutes,
// so the two sums are bit-identical) and run the same online softmax (one thread per
// head).  P goes to shared memory as bf16 and O_half += P V_half accumulates in TMEM
// (256 columns).
__global__ void __launch_bounds__(mla::kThreads, 1)
    attn_mla_tc(const AttnParams p, const __grid_constant__ CUtensorMap q_map) {
  using namespace mla;
  extern __shared__ uint8_t sm_raw_a[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)sm_raw_a + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* x_full = s_full + 2;
  uint64_t* sx_full = x_full + 2;
  uint64_t* p_full = sx_full + 2;
  uint64_t* p_free = p_full + 1;
  uint64_t* o_done = p_full + 2;
  uint64_t* q_full = p_full + 3;
  uint32_t* tmem_slot = (uint32_t*)(sm + kOffTmem);
  __shared__ int s_abort;
  __shared__ uint32_t s_mask[kStages];  // valid rows of the tile in each stage

  const int b = blockIdx.y;
  const int rank = (int)cluster_rank();  // == blockIdx.x & 1
  const int split = blockIdx.x >> 1;
  const int warp = warp_id(), lane = lane_id();
  const int T_all = (p.k + N - 1) / N;
  const int t0 = (int)(((long long)T_all * split) / p.nsplit);
  const int t1 = (int)(((long long)T_all * (split + 1)) / p.nsplit);
  const int my_tiles = t1 - t0;
  const uint32_t sbase = smem_u32(sm);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], kLoadWarps);  // one arrival per loader warp, after its copies
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&x_full[0], 128);  // the other CTA's softmax threads, remotely
    mbar_init(&x_full[1], 128);
    mbar_init(&sx_full[0], 128);  // this CTA's exchange threads: full S is in TMEM
    mbar_init(&sx_full[1], 128);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    mbar_init(q_full, 1);
    s_abort = 0;
    fence_mbar_init();
    if (p.early_q && my_tiles > 0) issue_q_load(sbase, &q_map, q_full, b, rank);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  // under programmatic dependent launch everything above overlaps the kernel before;
  // the selection, the rows and the outputs are touched only after it has finished
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem;          // columns [0, 256): O half
  const uint32_t tm_s = tmem + 256;    // columns [256, 320): S double buffer

  if (warp > kMmaWarp) {
    // ================= loaders: stage st holds tiles st, st + kStages, ... =================
    // Both warps of a stage resolve the tile's 32 rows (lane r -> row r).  The tile's
    // 32 x 40 16-byte chunks (this rank's five panels) are dealt over the stage's 64
    // threads in row-major order (consecutive threads, consecutive chunks of a row), each
    // copied with cp.async to its 128-byte-swizzled place; chunks of padding rows are
    // zeroed instead.  A thread waits for its own copies and makes them visible to the
    // tensor core (proxy fence); then its warp arrives on the stage's barrier.
    const int lw = warp - (kMmaWarp + 1);
    const int st = lw / kLoadWarps;
    const int t = (lw - st * kLoadWarps) * 32 + lane;  // thread within the stage
    const uint32_t stage = sbase + kOffKv + st * kStageBytes;
    const char* kv_base = (const char*)p.krows + rank * 4 * 128;  // first dim of panel 4r
    const long long row_bytes = p.row_stride * 2;
    // row of tile i for this lane; resolved one round ahead, so the two dependent loads
    // (selection, page table) overlap the wait for the stage
    auto tile_row = [&](int i) -> long long {
      const int j = (t0 + i) * N + lane;
      return (i < my_tiles && j < p.k) ? attn_row(p, b, p.sel[(size_t)b * p.k + j]) : -1;
    };
    long long row_next = tile_row(st);
    for (int i = st; i < my_tiles; i += kStages) {
      const long long row = row_next;
      row_next = tile_row(i + kStages);
      int go = 1;
      if (lane == 0) {  // one lane decides, so the warp stays converged
        go = (i < kStages) || mbar_wait(&kv_empty[st], ((i / kStages) - 1) & 1);
        if (*(volatile int*)&s_abort) go = 0;
        if (!go) s_abort = 1;
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) break;
      const uint32_t vmask = __ballot_sync(0xffffffffu, row >= 0);
#pragma unroll 5
      for (int it = 0; it < kChunksPerThread; ++it) {
        const int e = t + kLoadWarps * 32 * it;
        const int r = e / kChunksPerRow, c = e - r * kChunksPerRow;
        const long long rr = __shfl_sync(0xffffffffu, row, r);
        const uint32_t dst = stage + (c >> 3) * kKvPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        if (rr >= 0)
          cp_async_16(dst, kv_base + rr * row_bytes + c * 16);
        else
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0) : "memory");
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (t == 0) s_mask[st] = vmask;
        mbar_arrive(&kv_full[st]);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer: event driven =================
    // S(i) (this rank's panels) goes out whole once tile i has landed and S(i-2)'s
    // buffer is consumed; PV(i) as soon as P(i) is ready.  Neither blocks the other.
    if (lane == 0 && my_tiles > 0) {
      const uint32_t q_addr = sbase;
      const uint32_t p_addr = sbase + kOffP;
      const int nsp = s_panels(rank);
      const int lp0 = rank;  // first local panel used by S: rank 1 skips panel 4 (V only)
      if (!p.early_q) issue_q_load(sbase, &q_map, q_full, b, rank);
      bool ok = mbar_wait(q_full, 0);
      int ns = 0, npv = 0;
      uint64_t idle_since = 0;
      while (ok && npv < my_tiles) {
        bool progressed = false;
        if (npv < ns && mbar_test_wait(p_full, npv & 1)) {
          tc_fence_after();
          // this rank's V half is local panels 0-3 of the stage
          const uint32_t v = sbase + kOffKv + (npv % kStages) * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t ad = make_sdesc(p_addr + kk * 2 * 2048, 2048, 128, kSwizzleNone);
            const uint64_t bd = make_sdesc(v + kk * 16 * 128, kKvPanel, 1024, kSwizzle128);
            mma_bf16(tm_o, ad, bd, kIdescO, (npv > 0 || kk > 0));
          }
          tc_commit(&kv_empty[npv % kStages]);
          tc_commit(p_free);
          ++npv;
          progressed = true;
        }
        if (ns < my_tiles && ns < npv + 2 && mbar_test_wait(&kv_full[ns % kStages], (ns / kStages) & 1)) {
          tc_fence_after();
          const uint32_t kv = sbase + kOffKv + (ns % kStages) * kStageBytes + lp0 * kKvPanel;
          const uint32_t sb = tm_s + (ns & 1) * N;
#pragma unroll 1
          for (int pn = 0; pn < nsp; ++pn) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = make_sdesc(q_addr + pn * (H * 128) + kk * 32, 16, 1024, kSwizzle128);
              const uint64_t bd = make_sdesc(kv + pn * kKvPanel + kk * 32, 16, 1024, kSwizzle128);
              mma_bf16(sb, ad, bd, kIdescS, (pn | kk) != 0);
            }
          }
          tc_commit(&s_full[ns & 1]);
          ++ns;
          progressed = true;
        }
        if (progressed) {
          idle_since = 0;
        } else {
          const uint64_t now = globaltimer();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            flag(LS_DEV_TIMEOUT);
            ok = false;
          }
        }
      }
      if (!ok) s_abort = 1;
      tc_commit(o_done);
    }
  } else if (warp >= 4) {
    // ================= S exchange: warps 4..7, thread = head =================
    // Per tile: this rank's partial S from TMEM goes to the other CTA, the other rank's
    // partial is added, and the full S is written back over the partial in TMEM for the
    // softmax warps.  Runs a tile ahead of the softmax.
    const int q = warp & 3;
    const int h = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    // partials are stored chunk-major (chunk c of head h at c * 2048 + h * 16), so a
    // warp's 16-byte accesses are consecutive
    const uint32_t x_peer = dsmem_map(sbase + kOffX, (uint32_t)(rank ^ 1));
    const uint32_t xfull_peer = dsmem_map(smem_u32(x_full), (uint32_t)(rank ^ 1));
    for (int i = 0; i < my_tiles; ++i) {
      const int sb = i & 1;
      if (!mbar_wait(&s_full[sb], (i >> 1) & 1)) break;
      tc_fence_after();
      float s[N];
      tmem_ld32(tm_s + lane_off + sb * N, s);
#pragma unroll
      for (int c = 0; c < N / 4; ++c)
        st_cluster_v4(x_peer + sb * kXBytes + c * 2048 + h * 16, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      mbar_arrive_remote(xfull_peer + sb * 8);
      if (!mbar_wait_cluster(&x_full[sb], (i >> 1) & 1)) break;
#pragma unroll
      for (int c = 0; c < N / 4; ++c) {
        const float4 o = *(const float4*)(sm + kOffX + sb * kXBytes + c * 2048 + h * 16);
        s[4 * c] += o.x;
        s[4 * c + 1] += o.y;
        s[4 * c + 2] += o.z;
        s[4 * c + 3] += o.w;
      }
      tmem_st32(tm_s + lane_off + sb * N, s);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sx_full[sb]);
    }
  } else {
    // ================= softmax: warps 0..3, thread = head =================
    const int h = warp * 32 + lane;
    const float sl2 = p.scale * kLog2e;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < my_tiles; ++i) {
      const int st = i % kStages, sb = i & 1;
      // the loaders published the tile's valid rows with their kv_full arrivals
      if (!mbar_wait(&kv_full[st], (i / kStages) & 1)) { ok = false; break; }
      const uint32_t vmask = s_mask[st];
      // full S = both ranks' partials, summed by the exchange warps
      if (!mbar_wait(&sx_full[sb], (i >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float s[N];
      tmem_ld32(tm_s + lane_off + sb * N, s);
      float tmax = -INFINITY;
#pragma unroll
      for (int r = 0; r < N; ++r)
        if (vmask >> r & 1u) tmax = fmaxf(tmax, s[r]);
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
      float pr[N];
      float psum = 0.f;
#pragma unroll
      for (int r = 0; r < N; ++r) {
        pr[r] = (vmask >> r & 1u) ? exp2f(fmaf(s[r], sl2, -m_run)) : 0.f;
        psum += pr[r];
      }
      if (i >= 1 && !mbar_wait(p_free, (i - 1) & 1)) { ok = false; break; }
      // tcgen05.ld/st are warp-collective: the whole warp rescales when any lane must
      // (lanes that need not have factor 1)
      if (__any_sync(0xffffffffu, rescale)) {
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
      uint8_t* pbuf = sm + kOffP;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 two = __floats2bfloat162_rn(pr[c * 8 + 2 * e], pr[c * 8 + 2 * e + 1]);
          w[e] = *(uint32_t*)&two;
        }
        *(uint4*)(pbuf + h * 16 + c * 2048) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ---- epilogue
    bool fin = ok && my_tiles > 0 && mbar_wait(o_done, 0);
    fin = __all_sync(0xffffffffu, fin);  // the TMEM reads below are warp-collective
    if (fin) {
      tc_fence_after();
      const bool single = p.nsplit == 1;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      for (int c0 = 0; c0 < DVH; c0 += 32) {
        float v[32];
        tmem_ld32(tm_o + lane_off + c0, v);
        if (single) {
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
        } else {
          // layout [b][split][dim / 4][head][4]: a warp's store is 512 contiguous bytes
          float4* o = (float4*)p.part_o + (((size_t)b * p.nsplit + split) * (DV / 4) + (rank * DVH + c0) / 4) * H + h;
          const bool any = l_run > 0.f;
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            o[(size_t)(c / 4) * H] = any ? make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      if (rank == 0) {  // both ranks hold the same running max and sum
        if (single) {
          p.lse[(size_t)b * H + h] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        } else {
          float* ml = p.part_ml + (((size_t)b * p.nsplit + split) * H + h) * 2;
          ml[0] = l_run > 0.f ? m_run : -INFINITY;
          ml[1] = l_run;
        }
      }
    } else if (my_tiles == 0 && p.nsplit > 1) {
      float4* o = (float4*)p.part_o + (((size_t)b * p.nsplit + split) * (DV / 4) + rank * DVH / 4) * H + h;
      for (int c = 0; c < DVH / 4; ++c) o[(size_t)c * H] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rank == 0) {
        float* ml = p.part_ml + (((size_t)b * p.nsplit + split) * H + h) * 2;
        ml[0] = -INFINITY;
        ml[1] = 0.f;
      }
    }
  }
  // every warp must reach the barrier converged (the MMA warp's lane 0 arrives last).
  // The cluster-wide barrier also keeps this CTA's shared memory alive until the other
  // CTA has made its last remote write and arrival; only then may TMEM be released.
  __syncwarp();
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
// reads is a 512-byte run of the [dim / 4][head][4] layout; the 2 x nsplit 16-byte loads
// of a thread are independent of one another.
constexpr int kCombineThreads = 256;
__global__ void __launch_bounds__(kCombineThreads) attn_combine(const AttnParams p) {
  using namespace mla;
  griddep_wait();  // the partials come from the kernel before
  const int b = blockIdx.y;
  const int item = blockIdx.x * kCombineThreads + threadIdx.x;
  const int g = item / H, h = item - g * H, d0 = g * 8;
  const float* ml = p.part_ml + (size_t)b * p.nsplit * H * 2 + (size_t)h * 2;
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, ml[(size_t)s * H * 2]);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float Lsum = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int s = 0; s < p.nsplit; ++s) {
      const float l = ml[(size_t)s * H * 2 + 1];
      if (!(l > 0.f)) continue;
      const float wgt = exp2f(ml[(size_t)s * H * 2] - M);
      Lsum += wgt * l;
      const float4* po = (const float4*)p.part_o + (((size_t)b * p.nsplit + s) * (DV / 4) + d0 / 4) * H + h;
      const float4 x = po[0], y = po[H];
      acc[0] = fmaf(wgt, x.x, acc[0]); acc[1] = fmaf(wgt, x.y, acc[1]);
      acc[2] = fmaf(wgt, x.z, acc[2]); acc[3] = fmaf(wgt, x.w, acc[3]);
      acc[4] = fmaf(wgt, y.x, acc[4]); acc[5] = fmaf(wgt, y.y, acc[5]);
      acc[6] = fmaf(wgt, y.z, acc[6]); acc[7] = fmaf(wgt, y.w, acc[7]);
    }
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 two = __floats2bfloat162_rn(acc[2 * q] * inv, acc[2 * q + 1] * inv);
    w[q] = *(uint32_t*)&two;
  }
  *(uint4*)((__nv_bfloat16*)p.o + ((size_t)b * H + h) * DV + d0) = make_uint4(w[0], w[1], w[2], w[3]);
  if (d0 == 0) p.lse[(size_t)b * H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
}

}  // namespace ls
