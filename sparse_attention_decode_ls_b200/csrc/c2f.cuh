// a3. Coarse-to-fine indexer helpers (LeanSparse, abstract: coarse-to-fine indexing
// searches compact representations and retrieves original indexer keys only for
// candidate refinement).
//
//   build_summaries_kernel  per 64-token block: e4m3 [kmax | kmin] codes and a float32
//                           scale, rounded outward in exact (float64) arithmetic.
//   c2f_phase1_kernel       count / length of the blocks chosen for the tau0 pre-pass.
//   c2f_survivors_kernel    blocks whose bound (with margin) reaches tau0, compacted in
//                           ascending block order.
// The bound itself is the tcgen05 tile engine of the indexer (index_score.cuh) run
// over the summaries; the rescoring is the same engine over a list of pages.
#pragma once
#include "common.cuh"

namespace ls {

// Exact value of an e4m3 code (bias 7, subnormals m * 2^-9), as a double.
__device__ __forceinline__ double e4m3_exact(uint32_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  const double mag = e ? ldexp((double)(8 + m), e - 10) : ldexp((double)m, -9);
  return (c & 0x80u) ? -mag : mag;
}
// Finite e4m3 values in ascending order are indexed by o in [-126, 126].
__device__ __forceinline__ double e4m3_ord_value(int o) { return o >= 0 ? e4m3_exact(o) : -e4m3_exact(-o); }
__device__ __forceinline__ uint8_t e4m3_ord_code(int o) { return o >= 0 ? (uint8_t)o : (uint8_t)(0x80 | -o); }

struct SummParams {
  int B, max_pages, max_len, max_blocks;
  long long num_pages;
  const uint8_t* keys;   // [num_pages,64,128]
  const float* ks;       // [num_pages,64]
  const int* page_table;
  const int* lens;
  uint8_t* summ;         // [B,max_blocks,256]
  float* bscale;         // [B,max_blocks]
};

// grid (blocks, B), 128 threads (thread = dim).
__global__ void __launch_bounds__(128) build_summaries_kernel(const SummParams p) {
  __shared__ double red[4];
  const int j = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int L = p.lens[b];
  if (L < 0 || L > p.max_len || L > p.max_pages * 64 || ((L + 63) >> 6) > p.max_blocks) {
    if (j == 0 && d == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  if (j * 64 >= L) return;
  const int page = p.page_table[(size_t)b * p.max_pages + j];
  if (page < 0 || page >= p.num_pages) {
    if (d == 0) flag(LS_DEV_BOUNDS);
    return;
  }
  const int nt = min(64, L - j * 64);
  double kmax = -INFINITY, kmin = INFINITY;
  for (int t = 0; t < nt; ++t) {
    const size_t r = (size_t)page * 64 + t;
    const double v = (double)p.ks[r] * e4m3_exact(p.keys[r * 128 + d]);  // exact product
    kmax = fmax(kmax, v);
    kmin = fmin(kmin, v);
  }
  double a = fmax(fabs(kmax), fabs(kmin));
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmax(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((d & 31) == 0) red[d >> 5] = a;
  __syncthreads();
  const double amax = fmax(fmax(red[0], red[1]), fmax(red[2], red[3]));
  float bs = 1.f;
  if (amax > 0.0) {
    bs = __double2float_rn(amax / 448.0);
    if (448.0 * (double)bs < amax) bs = nextafterf(bs, INFINITY);
  }
  const double bsd = (double)bs;
  // smallest o with value(o) * bs >= kmax; largest o with value(o) * bs <= kmin
  int lo = -126, hi = 126;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;  // arithmetic shift: floor division
    if (e4m3_ord_value(mid) * bsd >= kmax) hi = mid;
    else lo = mid + 1;
  }
  const int o_up = lo;
  lo = -126;
  hi = 126;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (e4m3_ord_value(mid) * bsd <= kmin) lo = mid;
    else hi = mid - 1;
  }
  const int o_dn = lo;
  uint8_t* out = p.summ + ((size_t)b * p.max_blocks + j) * 256;
  out[d] = e4m3_ord_code(o_up);
  out[128 + d] = e4m3_ord_code(o_dn);
  if (d == 0) p.bscale[(size_t)b * p.max_blocks + j] = bs;
}

// After the top-(nb0) blocks by bound were chosen (ascending, -1 padded): how many
// were chosen and how many valid tokens they hold (a partial last block can only be
// the last entry).
__global__ void c2f_phase1_kernel(int B, int nb0, const int* lens, const int* blk, int* cnt, int* clen) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int L = max(0, lens[b]);
  const int NB = (L + 63) >> 6;
  const int c = min(nb0, NB);
  int len = c * 64;
  if (c > 0 && blk[(size_t)b * nb0 + c - 1] == NB - 1 && (L & 63)) len -= 64 - (L & 63);
  cnt[b] = c;
  clen[b] = len;
}

// One CTA per request: survivors = blocks j with ub_eff[j] >= tau0, ascending.
__global__ void __launch_bounds__(1024) c2f_survivors_kernel(int B, int max_blocks, int ub_stride, const int* lens,
                                                             const float* ub_eff, const float* tau0, int* surv,
                                                             int* n_surv, int* clen) {
  __shared__ unsigned long long scan_tmp[32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int L = max(0, lens[b]);
  const int NB = min((L + 63) >> 6, max_blocks);
  const float t = tau0[b];
  const int per = (NB + 1023) / 1024;
  const int j0 = min(NB, tid * per), j1 = min(NB, j0 + per);
  uint32_t c = 0;
  for (int j = j0; j < j1; ++j) c += ub_eff[(size_t)b * ub_stride + j] >= t;
  unsigned long long tot;
  uint32_t o = (uint32_t)block_excl_scan_u64(c, scan_tmp, &tot);
  for (int j = j0; j < j1; ++j)
    if (ub_eff[(size_t)b * ub_stride + j] >= t) surv[(size_t)b * max_blocks + (o++)] = j;
  if (tid == 0) {
    const int n = (int)tot;
    n_surv[b] = n;
    int len = n * 64;
    // the partial last block, if it survived, is the last entry (its tail is not data)
    if (n > 0 && (L & 63) && ub_eff[(size_t)b * ub_stride + NB - 1] >= t) len -= 64 - (L & 63);
    clen[b] = len;
  }
}

}  // namespace ls
