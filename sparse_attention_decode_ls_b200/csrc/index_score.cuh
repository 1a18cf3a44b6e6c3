// a1. Indexer score kernels.
//
// score[b][s] = key_scale[s] * sum_h (w[b][h] * q_scale[b][h]) * ReLU(q8[b][h] . k8[s])
//
// (the DSA lightning-indexer form; LeanSparse, abstract, names indexer keys and
// indexer scores).  Two kernels:
//   * index_score_tc   tcgen05 fp8 MMA.  A 128-row tile of keys (two 64-token pages,
//                      TMA-loaded with 128-byte swizzle) is the A operand (M = 128
//                      tokens), the query's heads are the B operand (N = 64), so each
//                      epilogue thread owns one token's TMEM row and reduces the heads
//                      in registers: ReLU, head weights and the token scale are fused.
//                      The same tile engine also computes the coarse-to-fine block
//                      bound (K = 256 bytes: [kmax | kmin] rows against [q+ | q-]).
//   * index_score_simt CUDA cores, fp32 (and an e4m3 cross-check variant).
#pragma once
#include "common.cuh"

namespace ls {

// =====================================================================================
// CUDA-core kernel: one 64-token page per CTA, 256 threads (token = tid % 64,
// head group = tid / 64).
// =====================================================================================
struct IdxSimtParams {
  int B, H, D, max_pages, max_len;
  long long num_pages;
  const void* q;
  const float* qs;
  const void* w;
  int w_bf16;
  const void* keys;
  const float* ks;
  const int* page_table;
  const int* lens;
  float* out;
};

template <bool E4M3>
__global__ void __launch_bounds__(256) index_score_simt(IdxSimtParams p) {
  extern __shared__ __align__(16) float sm_simt[];
  const int b = blockIdx.y, lp = blockIdx.x, tid = threadIdx.x;
  const int L = p.lens[b];
  if (L < 0 || L > p.max_len || L > p.max_pages * 64) {
    if (lp == 0 && tid == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  if (lp * 64 >= L) return;
  const int page = p.page_table[(size_t)b * p.max_pages + lp];
  if (page < 0 || page >= p.num_pages) {
    if (tid == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  const int H = p.H, D = p.D, Dp = D + 1;
  float* q_s = sm_simt;             // [H][D]
  float* k_s = q_s + H * D;         // [64][D+1]
  float* coef = k_s + 64 * Dp;      // [H]
  float* part = coef + H;           // [4][64]
  for (int i = tid; i < H * D; i += 256) {
    const size_t gi = (size_t)b * H * D + i;
    q_s[i] = E4M3 ? e4m3_to_float(((const uint8_t*)p.q)[gi]) : ((const float*)p.q)[gi];
  }
  for (int h = tid; h < H; h += 256) {
    const size_t gi = (size_t)b * H + h;
    float wv = p.w_bf16 ? __bfloat162float(((const __nv_bfloat16*)p.w)[gi]) : ((const float*)p.w)[gi];
    coef[h] = E4M3 ? wv * p.qs[gi] : wv;
  }
  for (int i = tid; i < 64 * D; i += 256) {
    const int t = i / D, d = i - t * D;
    const size_t gi = ((size_t)page * 64 + t) * D + d;
    k_s[t * Dp + d] = E4M3 ? e4m3_to_float(((const uint8_t*)p.keys)[gi]) : ((const float*)p.keys)[gi];
  }
  __syncthreads();
  const int t = tid & 63, g = tid >> 6;
  float acc = 0.f;
  for (int h = g; h < H; h += 4) {
    float dot = 0.f;
    const float* qh = q_s + h * D;
    const float* kt = k_s + t * Dp;
    for (int d = 0; d < D; ++d) dot = fmaf(qh[d], kt[d], dot);
    acc = fmaf(coef[h], fmaxf(dot, 0.f), acc);
  }
  part[g * 64 + t] = acc;
  __syncthreads();
  if (g == 0) {
    const int s = lp * 64 + t;
    if (s < L) {
      float v = part[t] + part[64 + t] + part[128 + t] + part[192 + t];
      if (E4M3) v *= p.ks[(size_t)page * 64 + t];
      p.out[(size_t)b * p.max_len + s] = v;
    }
  }
}

// =====================================================================================
// tcgen05 kernel
// =====================================================================================
struct IdxTcParams {
  int mode;              // 0: paged keys (dense, or a list of logical pages); 1: block summaries
  int B, max_pages, max_len, max_blocks, ctas_per_req;
  long long num_pages;
  const uint8_t* q8;     // [B,64,128]
  const float* qs;       // [B,64]
  const void* w;         // [B,64]
  int w_bf16;
  const float* row_scale;  // mode 0: key scale pool [num_pages*64]; mode 1: block scale [B*max_blocks]
  const int* page_table;
  const int* lens;
  const int* unit_list;    // mode 0 list: [B,list_stride] logical pages (ascending); NULL = every page
  const int* unit_count;   // [B] length of each list
  int list_stride;
  float* out;              // [B,out_stride]
  long long out_stride;
  float* out_plain;        // mode 1: bound without margin, [B,max_blocks] (may be NULL)
  float eps_rel;           // mode 1: margin relative to the block magnitude bound
  int staged;              // mode 0 list: entries [unit_base, unit_base + stage_cap) of the list,
  int unit_base;           //   whose keys were copied to staging units b * stage_cap + (entry -
  int stage_cap;           //   unit_base) of the pool (key_pool / row_scale point at the staging)
  int* clear;              // optional [B]: set to 0 (the top-k's per-request count, which the
                           //   top-k adds up after this kernel has finished)
  // optional candidate filter (mode 0 over whole requests): see the epilogue
  int* filt;               // [B][kFiltInts]: zeroed by the top-k that reads them (any contents
                           //   give exact results; stale ones can only cost the fast path)
  int* cand_cnt;           // [B][ctas_per_req * 4] candidates each epilogue warp found
  int* cand_pos;           // [B][ctas_per_req * 4][kCandPerWarp] their positions
  float* cand_score;       // [B][ctas_per_req * 4][kCandPerWarp] and scores
  int filt_k;              // the k of the selection the candidates serve
};

// FILT: the instance that also keeps candidate lists (key scoring in the decode step); its
// filter state takes the room of one pipeline stage.
template <int KP, int NCOL, bool FILT = false>
struct IdxTc {
  static constexpr int kThreads = 192;                 // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
  static constexpr int kPanel = 128 * 128;             // one 128-row x 128-byte K panel
  static constexpr int kStageBytes = KP * kPanel;
  static constexpr int kStages = (KP == 1) ? (FILT ? 5 : 6) : 3;
  static constexpr int kAcc = 256 / NCOL;              // accumulators in 256 TMEM columns
  static constexpr int kBBytes = KP * NCOL * 128;
  static constexpr int kOffB = kStages * kStageBytes;
  static constexpr int kOffScale = kOffB + kBBytes;                  // [kStages][128] row scales
  static constexpr int kOffMeta = kOffScale + kStages * 128 * 4;     // [kStages][2] logical unit ids
  static constexpr int kOffCoef = kOffMeta + ((kStages * 8 + 15) & ~15);
  static constexpr int kOffBar = kOffCoef + NCOL * 4 + 16;
  static constexpr int kNumBars = 2 * kStages + 2 * kAcc + 1;  // + b_ready
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  // candidate filter (key scoring only): the scores of the tiles scored before the threshold
  // is known, and each row's scores that passed it with their tile numbers
  static constexpr int kFiltBacklog = FILT ? 16 : 0;   // tiles
  static constexpr int kRowCand = FILT ? 8 : 0;        // passing scores kept per row
  static constexpr int kOffBl = (kOffTmem + 16 + 15) & ~15;
  static constexpr int kOffLcs = kOffBl + kFiltBacklog * 128 * 4;
  static constexpr int kOffLct = kOffLcs + 128 * kRowCand * 4;
  static constexpr int kSmem = 1024 + kOffLct + 128 * kRowCand * 2;  // +1024: runtime alignment slack
  static constexpr uint32_t kIdesc = make_idesc(0 /*e4m3*/, 128, NCOL, false, false);
};

// Row coordinate (in 64-row units of the tensor map) of one unit, or -1 if the unit
// has no data to load.
__device__ __forceinline__ int idx_unit_row(const IdxTcParams& p, int b, int u, int* lp_out) {
  if (p.mode == 1) {
    *lp_out = u;
    return b * p.max_blocks + u * 64;
  }
  int lp = p.unit_list ? p.unit_list[(size_t)b * p.list_stride + p.unit_base + u] : u;
  *lp_out = lp;
  if (lp < 0 || lp >= p.max_pages) return -1;
  if (p.staged) return (b * p.stage_cap + u) * 64;
  const int page = p.page_table[(size_t)b * p.max_pages + lp];
  if (page < 0 || page >= p.num_pages) return -1;
  return page * 64;
}

// The key-scoring instance (KP = 1) runs two CTAs per SM, so it must stay within 168 registers.
template <int KP, int NCOL, bool FILT = false>
__global__ void __launch_bounds__(192, KP == 1 ? 2 : 1)
    index_score_tc(const IdxTcParams p, const __grid_constant__ CUtensorMap tmap) {
  using C = IdxTc<KP, NCOL, FILT>;
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)sm_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = sm;
  uint8_t* sB = sm + C::kOffB;
  float* s_scale = (float*)(sm + C::kOffScale);
  int* s_meta = (int*)(sm + C::kOffMeta);
  float* coef = (float*)(sm + C::kOffCoef);
  float* gmag = coef + NCOL;  // mode 1: sum_h |w'_h| * sum_d |q8_hd|
  uint64_t* bars = (uint64_t*)(sm + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* accf = bars + 2 * C::kStages;
  uint64_t* acce = accf + C::kAcc;
  uint64_t* b_ready = acce + C::kAcc;
  uint32_t* tmem_slot = (uint32_t*)(sm + C::kOffTmem);
  float* s_bl = (float*)(sm + C::kOffBl);        // [kFiltBacklog][128]
  float* s_lcs = (float*)(sm + C::kOffLcs);      // [128][kRowCand]
  uint16_t* s_lct = (uint16_t*)(sm + C::kOffLct);
  __shared__ int s_abort;
  __shared__ __align__(16) int s_fpoll[4][4];  // each epilogue warp's copy of the filter's words
  __shared__ __align__(8) uint64_t s_pbar[4];  // each epilogue warp's copy of the request's words

  const int b = blockIdx.y, cta = blockIdx.x, tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  griddep_launch_dependents();  // the next kernel may be scheduled now; it waits for this one
  if (p.clear && cta == 0 && tid == 0) p.clear[b] = 0;
  const int L = p.lens[b];
  const bool len_ok = L >= 0 && L <= p.max_len && L <= p.max_pages * 64;
  if (!len_ok) {
    if (cta == 0 && tid == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  int n_units;
  if (p.mode == 1) {
    if (((L + 63) >> 6) > p.max_blocks) {
      if (cta == 0 && tid == 0) flag(LS_DEV_BOUNDS);
      return;
    }
    n_units = (((L + 63) >> 6) + 63) >> 6;
  } else if (p.unit_list) {
    n_units = p.unit_count[b];
    if (n_units < 0 || n_units > p.list_stride) {
      if (cta == 0 && tid == 0) flag(LS_DEV_BOUNDS);
      return;
    }
    if (p.staged) n_units = min(max(n_units - p.unit_base, 0), p.stage_cap);  // this pass's window
  } else {
    n_units = (L + 63) >> 6;
  }
  const int n_tiles = (n_units + 1) >> 1;
  const int t_begin = (int)(((long long)n_tiles * cta) / p.ctas_per_req);
  const int t_end = (int)(((long long)n_tiles * (cta + 1)) / p.ctas_per_req);
  const int my_tiles = t_end - t_begin;
  if (my_tiles <= 0) {
    // a CTA without tiles has no candidates (the top-k reads every CTA's count)
    if (FILT && p.filt && p.mode == 0 && !p.unit_list && tid < 4) p.cand_cnt[((size_t)b * p.ctas_per_req + cta) * 4 + tid] = 0;
    return;
  }

  // ---- query side: B operand in 128-byte-swizzled K-major layout, coefficients and, for
  // the bound, the magnitude used by the margin.  The epilogue warps build it while the
  // producer's first loads are in flight; the MMA waits for it on b_ready.
  const uint8_t* q8 = p.q8 + (size_t)b * 64 * 128;
  auto build_query_side = [&](int et) {  // et: epilogue thread index in [0, 128)
  for (int i = et; i < NCOL * 8 * KP; i += 128) {
    // i enumerates 16-byte chunks: panel pk, row n, chunk j
    const int pk = i / (NCOL * 8);
    const int rem = i - pk * NCOL * 8;
    const int n = rem >> 3, j = rem & 7;
    uint4 v;
    if (KP == 1) {
      v = *(const uint4*)(q8 + n * 128 + j * 16);
    } else {
      // rows 0..63: [q+ | q-], rows 64..127: [q- | q+]  (q+ keeps codes with clear sign bit)
      const int h = n & 63;
      const bool want_pos = ((n < 64) == (pk == 0));
      uint4 raw = *(const uint4*)(q8 + h * 128 + j * 16);
      uint32_t* r = (uint32_t*)&raw;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t x = r[e], out = 0;
#pragma unroll
        for (int by = 0; by < 4; ++by) {
          uint32_t c = (x >> (8 * by)) & 0xFFu;
          bool neg = (c & 0x80u) != 0;
          if (neg != want_pos) out |= c << (8 * by);
        }
        r[e] = out;
      }
      v = raw;
    }
    const int off = pk * NCOL * 128 + n * 128 + ((j ^ (n & 7)) << 4);
    *(uint4*)(sB + off) = v;
  }
  if (et < 64) {
    const size_t gi = (size_t)b * 64 + et;
    const float wv = p.w_bf16 ? __bfloat162float(((const __nv_bfloat16*)p.w)[gi]) : ((const float*)p.w)[gi];
    const float wq = wv * p.qs[gi];
    if (NCOL == 64) {
      coef[et] = wq;
    } else {
      coef[et] = fmaxf(wq, 0.f);
      coef[64 + et] = fminf(wq, 0.f);
    }
  }
  if (p.mode == 1 && et < 32) {
    // magnitude bound used for the pruning margin
    float acc = 0.f;
    for (int h = et; h < 64; h += 32) {
      float s = 0.f;
      for (int d = 0; d < 128; ++d) s += fabsf(e4m3_to_float(q8[h * 128 + d]));
      const size_t gi = (size_t)b * 64 + h;
      const float wv = p.w_bf16 ? __bfloat162float(((const __nv_bfloat16*)p.w)[gi]) : ((const float*)p.w)[gi];
      acc += fabsf(wv * p.qs[gi]) * s;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (et == 0) gmag[0] = acc;
  }
  fence_proxy_async_smem();
  };
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 128);  // MMA commit + every epilogue thread
    }
    for (int a = 0; a < C::kAcc; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 128);
    }
    mbar_init(b_ready, 128);
    s_abort = 0;
    for (int w = 0; w < 4; ++w) mbar_init(&s_pbar[w], 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    const uint64_t stream_pol = l2_evict_first_policy();  // keys and scales are read once
    // Per tile: the keys of its two 64-row units (TMA, 128-byte swizzle) and, for keys,
    // their 64 token scales (bulk copy) into the stage, plus each unit's logical id.
    // A stage is released only when the MMA has consumed it and the epilogue has read
    // its scales and ids.
    // The warp fetches the rows of 32 units (16 tiles) at a time, so the page-table
    // reads are off the issue path; lane 0 waits for free stages and issues the copies.
    if (lane == 0) prefetch_tmap(&tmap);
    int issued = 0;
    bool go = true;
    for (int i0 = 0; go && i0 < my_tiles; i0 += 16) {
      const int u_lane = 2 * (t_begin + i0) + lane;
      int row_l = -1, lp_l = -1;
      if (u_lane < n_units) {
        row_l = idx_unit_row(p, b, u_lane, &lp_l);
        if (row_l < 0) {
          flag(LS_DEV_BOUNDS);
          lp_l = -1;
        }
      }
      const int nt = min(16, my_tiles - i0);
      for (int ii = 0; ii < nt; ++ii) {
        const int i = i0 + ii;
        const int st = i % C::kStages;
        const int row0 = __shfl_sync(0xffffffffu, row_l, 2 * ii);
        const int row1 = __shfl_sync(0xffffffffu, row_l, 2 * ii + 1);
        const int lp0 = __shfl_sync(0xffffffffu, lp_l, 2 * ii);
        const int lp1 = __shfl_sync(0xffffffffu, lp_l, 2 * ii + 1);
        int ok_i = 1;
        if (lane == 0) {
          if (i >= C::kStages && !mbar_wait(&empty[st], ((i / C::kStages) - 1) & 1)) ok_i = 0;
          if (*(volatile int*)&s_abort) ok_i = 0;
          if (!ok_i) {
            s_abort = 1;
          } else {
            constexpr uint32_t kUnitBytes = KP * 64 * 128;
            const uint32_t extra = p.mode == 0 ? 256u : 0u;
            s_meta[st * 2 + 0] = lp0;
            s_meta[st * 2 + 1] = lp1;
            const uint32_t bytes = (row0 >= 0 ? kUnitBytes + extra : 0u) + (row1 >= 0 ? kUnitBytes + extra : 0u);
            mbar_arrive_expect_tx(&full[st], bytes);
            const uint32_t dst = smem_u32(sA + st * C::kStageBytes);
            const int rows[2] = {row0, row1};
            for (int uu = 0; uu < 2; ++uu) {
              if (rows[uu] < 0) continue;
              for (int pk = 0; pk < KP; ++pk)
                tma_load_2d_hint(dst + pk * C::kPanel + uu * 64 * 128, &tmap, &full[st], pk * 128, rows[uu],
                                 stream_pol);
              if (p.mode == 0)
                bulk_load_hint(smem_u32(s_scale + st * 128 + uu * 64), p.row_scale + rows[uu], 256, &full[st],
                               stream_pol);
            }
          }
        }
        ok_i = __shfl_sync(0xffffffffu, ok_i, 0);
        if (!ok_i) {
          go = false;
          break;
        }
        ++issued;
      }
    }
    // never leave with copies in flight: wait for every stage still owned by TMA
    if (lane == 0) {
      const int first = issued > C::kStages ? issued - C::kStages : 0;
      for (int i = first; i < issued; ++i) mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t b_base = smem_u32(sB);
      const bool have_b = mbar_wait(b_ready, 0);
      if (!have_b) s_abort = 1;
      for (int i = 0; have_b && i < my_tiles; ++i) {
        const int st = i % C::kStages, a = i % C::kAcc;
        if (!mbar_wait(&full[st], (i / C::kStages) & 1)) { s_abort = 1; break; }
        if (i >= C::kAcc && !mbar_wait(&acce[a], ((i / C::kAcc) - 1) & 1)) { s_abort = 1; break; }
        if (*(volatile int*)&s_abort) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + st * C::kStageBytes);
#pragma unroll
        for (int pk = 0; pk < KP; ++pk) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc(a_base + pk * C::kPanel + kk * 32, 16, 1024, kSwizzle128);
            const uint64_t bd = make_sdesc(b_base + pk * NCOL * 128 + kk * 32, 16, 1024, kSwizzle128);
            mma_f8(tmem + a * NCOL, ad, bd, C::kIdesc, (pk | kk) != 0);
          }
        }
        tc_commit(&empty[st]);
        tc_commit(&accf[a]);
      }
    }
  } else {
    // ================= epilogue: warps 2..5, thread = tile row =================
    build_query_side(tid - 64);
    asm volatile("bar.sync 1, 128;" ::: "memory");  // coefficients visible to all epilogue warps
    mbar_arrive(b_ready);
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int rr = r & 63;
    const float mag = (p.mode == 1) ? gmag[0] : 0.f;
    const int nb = (L + 63) >> 6;
    // ---- candidate filter.  Besides every score, the scores at or above a per-request
    // threshold tau go to candidate lists, so that the top-k can select among a few thousand
    // entries instead of the whole request.  tau comes from the request's own scores: each
    // epilogue warp takes the j-th largest score of its 32 rows of its first tile (j ~ 64 k / L,
    // so that about 2k scores of the request lie above such a statistic) and adds it, as an
    // order-preserving key, with a count into one 64-bit word of the request; the first warp of
    // CTA 0, once it sees the word hold 32 of them (fewer for a short request), sets tau to the
    // mean of the keys it saw.  The tile loop never waits on memory for this: the additions
    // return nothing, and each warp learns of tau from an asynchronous copy of the request's
    // words whose barrier it tests without blocking; a load issued then is checked at the end
    // against the tau it used.  Until tau is known, every
    // score also goes to shared memory; then those tiles are checked from there.  A row keeps
    // the scores that passed (with their tile numbers) in shared memory, and each epilogue warp
    // writes its rows' candidates to a list of its own after its last tile.  Any tau gives an
    // exact result: the top-k uses the lists only when at least k scores passed (then the k-th
    // largest is among them) and every list is complete; a warp that did not see tau within
    // kFiltBacklog tiles (or saw another tau than the one set), a row or list that ran full or
    // an aborted CTA marks the request incomplete.
    const bool filt = FILT && p.filt != nullptr && p.mode == 0 && !p.unit_list;
    int* fctl = filt ? p.filt + (size_t)b * kFiltInts : nullptr;
    const int n_need = 4 * min(min(p.ctas_per_req, n_tiles), 8);  // statistics that set tau
    const int fj = filt ? min(8, max(1, (int)((64LL * p.filt_k + L - 1) / max(L, 1)))) : 1;
    const bool publisher = filt && cta == 0 && wq == 0;
    bool tau_known = false, gave_up = false;
    float tau = 0.f;
    int nk = 0;                            // this row's passing scores
    unsigned long long tau_check = 0;      // lane 0: the request's tau word, loaded when seen
    uint32_t poll_ph = 0;
    bool poll_inflight = false;            // lane 0: a copy of the request's words in flight
    float* my_lcs = s_lcs + r * C::kRowCand;
    uint16_t* my_lct = s_lct + r * C::kRowCand;
    auto keep = [&](int t, float v) {
      if (nk < C::kRowCand) {
        my_lcs[nk] = v;
        my_lct[nk] = (uint16_t)t;
      }
      ++nk;
    };
    auto look = [&]() {  // lane 0: copy the request's first 16 bytes in (through the load path)
      cp_async_16(smem_u32(&s_fpoll[wq][0]), fctl);
      cp_async_mbar_arrive(&s_pbar[wq]);
      poll_inflight = true;
    };
    if (filt && lane == 0) look();
    for (int i = 0; i < my_tiles; ++i) {
      const int st = i % C::kStages, a = i % C::kAcc;
      const int tile = t_begin + i;
      const int u = 2 * tile + (r >> 6);
      // the stage's unit ids and scales (written by the producer / TMA) -- acquire them
      if (!mbar_wait(&full[st], (i / C::kStages) & 1)) { s_abort = 1; break; }
      const int lp = s_meta[st * 2 + (r >> 6)];
      bool valid = false;
      float scale = 0.f;
      long long out_idx = 0;
      if (p.mode == 1) {
        const int j = u * 64 + rr;
        if (lp >= 0 && j < nb) {
          valid = true;
          scale = p.row_scale[(size_t)b * p.max_blocks + j];
          out_idx = j;
        }
      } else if (lp >= 0 && lp * 64 + rr < L) {
        valid = true;
        scale = s_scale[st * 128 + r];
        out_idx = p.unit_list ? (long long)(p.unit_base + u) * 64 + rr : (long long)lp * 64 + rr;
      }
      // the stage's metadata is read: the producer may refill it once the MMA has read its keys
      // too (the MMA's commit is the stage's other arrival), so the loads need not wait for
      // this tile's epilogue
      mbar_arrive(&empty[st]);
      if (!mbar_wait(&accf[a], (i / C::kAcc) & 1)) { s_abort = 1; break; }
      tc_fence_after();
      // four independent partial sums (fixed order: the result is the same for a token
      // wherever it is scored)
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
      const uint32_t tbase = tmem + ((uint32_t)(wq * 32) << 16) + a * NCOL;
#pragma unroll
      for (int c0 = 0; c0 < NCOL; c0 += 64) {
        float v[64];
        tmem_ld64(tbase + c0, v);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 cf = *(const float4*)(coef + c0 + c);
          acc0 = fmaf(cf.x, fmaxf(v[c], 0.f), acc0);
          acc1 = fmaf(cf.y, fmaxf(v[c + 1], 0.f), acc1);
          acc2 = fmaf(cf.z, fmaxf(v[c + 2], 0.f), acc2);
          acc3 = fmaf(cf.w, fmaxf(v[c + 3], 0.f), acc3);
        }
      }
      const float sum = (acc0 + acc1) + (acc2 + acc3);
      tc_fence_before();
      mbar_arrive(&acce[a]);
      if (valid) {
        float* o = p.out + (size_t)b * p.out_stride;
        if (p.mode == 1) {
          const float ub = sum * scale;
          if (p.out_plain) p.out_plain[(size_t)b * p.max_blocks + out_idx] = ub;
          o[out_idx] = ub + p.eps_rel * 448.f * scale * mag;
        } else {
          o[out_idx] = sum * scale;
        }
      }
      if (filt) {
        const float sc = valid ? sum * scale : -INFINITY;
        if (!tau_known) {  // (giving up sets tau_known with tau = +inf: one test per tile after)
          s_bl[i * 128 + r] = sc;
          if (i == 0) {
            // this warp's statistic: the fj-th largest score of its rows of the first tile; its
            // key goes into the request's word with a count from bit 48 (the sum of the keys
            // below; at most 2^16 additions)
            float v = sc, kth = -INFINITY;
            for (int q = 0; q < fj; ++q) {
              float mx = v;
#pragma unroll
              for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
              kth = mx;
              const uint32_t own = __ballot_sync(0xffffffffu, v == mx);
              if (lane == __ffs(own) - 1) v = -INFINITY;  // take one copy of the maximum out
            }
            if (lane == 0) atomicAdd((unsigned long long*)(fctl + kFiltStat), (1ull << 48) | float_key(kth));
          }
          int f = 0;
          float t = 0.f;
          if (lane == 0 && poll_inflight && mbar_test_wait(&s_pbar[wq], poll_ph)) {
            poll_ph ^= 1u;
            poll_inflight = false;
            f = *(volatile int*)&s_fpoll[wq][kFiltReady];
            t = *(volatile float*)&s_fpoll[wq][kFiltTau];
            const unsigned long long sw = *(volatile unsigned long long*)&s_fpoll[wq][kFiltStat];
            if (f) {
              tau_check = ld_relaxed_gpu_u64(fctl + kFiltReady);  // looked at after the last tile
            } else if (publisher && (int)(sw >> 48) >= n_need) {
              // enough statistics: tau = the mean of their keys, published once
              const unsigned long long cnt = sw >> 48;
              t = key_float((uint32_t)((sw & ((1ull << 48) - 1)) / cnt));
              tau_check = ((unsigned long long)__float_as_uint(t) << 32) | 1ull;
              atomicExch((unsigned long long*)(fctl + kFiltReady), tau_check);
              f = 1;
            } else {
              look();
            }
          }
          f = __shfl_sync(0xffffffffu, f, 0);
          if (f) {
            tau = __shfl_sync(0xffffffffu, t, 0);
            tau_known = true;
            // the tiles scored before (this one included), from shared memory
            for (int t2 = 0; t2 <= i; ++t2) {
              const float v = s_bl[t2 * 128 + r];
              if (v >= tau && v != -INFINITY) keep(t2, v);
            }
          } else if (i + 1 >= C::kFiltBacklog) {
            gave_up = true;  // too many tiles to keep: this request's lists stay incomplete
            tau_known = true;
            tau = INFINITY;
          }
        } else if (sc >= tau && valid) {
          keep(i, sc);
        }
      }
    }
    if (filt) {
      // the statistic if not yet looked at, then the rows' candidates into this warp's list
      const bool aborted = *(volatile int*)&s_abort != 0;
      bool bad = __any_sync(0xffffffffu, nk > C::kRowCand) || !tau_known || gave_up || aborted;
      if (lane == 0) {
        if (poll_inflight) mbar_wait(&s_pbar[wq], poll_ph);  // the copy lands before the CTA ends
        if (tau_known && !gave_up && (!(uint32_t)tau_check || (tau_check >> 32) != __float_as_uint(tau)))
          bad = true;
      }
      bad = __shfl_sync(0xffffffffu, (int)bad, 0) != 0;
      const size_t wlist = (((size_t)b * p.ctas_per_req + cta) * 4 + wq) * kCandPerWarp;
      int wcnt = 0;
      if (!bad) {
        const int mine = min(nk, C::kRowCand);
        const int rounds = __reduce_max_sync(0xffffffffu, (uint32_t)mine);
        for (int q = 0; q < rounds; ++q) {
          const bool take = q < mine;
          const uint32_t m = __ballot_sync(0xffffffffu, take);
          const int o = wcnt + __popc(m & ((1u << lane) - 1u));
          if (take && o < kCandPerWarp) {
            p.cand_pos[wlist + o] = (2 * (t_begin + (int)my_lct[q]) + (r >> 6)) * 64 + rr;
            p.cand_score[wlist + o] = my_lcs[q];
          }
          wcnt += __popc(m);
        }
      }
      if (lane == 0) {
        if (bad || wcnt > kCandPerWarp) fctl[kFiltIncomplete] = 1;
        p.cand_cnt[((size_t)b * p.ctas_per_req + cta) * 4 + wq] = min(wcnt, kCandPerWarp);
      }
    }
  }
  // every warp must reach the barrier converged (the MMA warp's lane 0 arrives last);
  // only then may TMEM be released
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Host-resident keys: copy the keys (64 x 128 e4m3 = 8 KB) and token scales (256 B) of
// list entries [base, base + cap) of each request from pinned host memory (zero-copy
// reads over the host link) to staging units b * cap + (entry - base).  grid (ctas, B),
// 128 threads; a warp per block, all of its 16-byte loads in flight before any store.
struct FetchParams {
  int B, max_pages, list_stride, base, cap;
  long long num_pages;
  const uint8_t* host_keys;   // [num_pages, 64, 128]
  const float* host_scales;   // [num_pages, 64]
  const int* page_table;      // [B, max_pages]
  const int* list;            // [B, list_stride] logical blocks
  const int* count;           // [B]
  uint8_t* stage_keys;        // [B * cap, 64, 128]
  float* stage_scales;        // [B * cap, 64]
};

__global__ void __launch_bounds__(128) fetch_blocks_kernel(const FetchParams p) {
  const int b = blockIdx.y;
  const int cnt = p.count[b];
  if (cnt < 0 || cnt > p.list_stride) return;  // flagged by the scoring kernel
  const int n = min(max(cnt - p.base, 0), p.cap);
  const int lane = lane_id();
  for (int u = blockIdx.x * 4 + warp_id(); u < n; u += gridDim.x * 4) {
    const int lp = p.list[(size_t)b * p.list_stride + p.base + u];
    if (lp < 0 || lp >= p.max_pages) continue;  // flagged by the scoring kernel, which skips it
    const int page = p.page_table[(size_t)b * p.max_pages + lp];
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) flag(LS_DEV_BOUNDS);
      continue;
    }
    const uint4* src = (const uint4*)(p.host_keys + (size_t)page * 8192);
    uint4* dst = (uint4*)(p.stage_keys + ((size_t)b * p.cap + u) * 8192);
    uint4 v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = src[j * 32 + lane];
    uint4 sc = make_uint4(0, 0, 0, 0);
    if (lane < 16) sc = ((const uint4*)(p.host_scales + (size_t)page * 64))[lane];
#pragma unroll
    for (int j = 0; j < 16; ++j) dst[j * 32 + lane] = v[j];
    if (lane < 16) ((uint4*)(p.stage_scales + ((size_t)b * p.cap + u) * 64))[lane] = sc;
  }
}

}  // namespace ls
