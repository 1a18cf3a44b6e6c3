// Host side of the C ABI declared in include/ls.h: argument validation, launch
// configuration, TMA descriptors, workspace carving and the decode-step orchestration.
// The kernels are in the .cuh files included below (one translation unit, so the
// device status word is a single symbol).
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "attn.cuh"
#include "c2f.cuh"
#include "common.cuh"
#include "hotbuf.cuh"
#include "cp.cuh"
#include "topk_row.cuh"
#include "index_score.cuh"
#include "topk.cuh"

#define LS_VERSION_STRING "sparse_attention_decode_ls_b200 0.1 (sm_100a)"

namespace {

thread_local std::string g_last_error;

ls_status fail(ls_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

ls_status ok() {
  g_last_error.clear();
  return LS_OK;
}

ls_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return LS_OK;
}

#define LS_REQUIRE(cond, ...)                                   \
  do {                                                          \
    if (!(cond)) return fail(LS_ERR_INVALID_ARG, __VA_ARGS__);  \
  } while (0)
#define LS_TRY(expr)                   \
  do {                                 \
    ls_status _s = (expr);             \
    if (_s != LS_OK) return _s;        \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// ---- per-device cached properties -------------------------------------------------
// Per-device caches below hold this many devices; a higher ordinal is refused
// (LS_ERR_UNSUPPORTED or cudaErrorInvalidDevice), never folded onto a lower one.
constexpr int kMaxDevices = 64;

int device_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < kMaxDevices;
  int v = cached ? cache[dev].load() : 0;
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    if (cached) cache[dev].store(v);
  }
  return v;
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
cudaError_t allow_smem(K kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  if (done.load() & bit) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

// Ask for the SM's full shared-memory carve-out for a kernel that needs little of it: an
// SM's split between L1 and shared memory changes only when the SM is idle, so a small
// kernel that left its SMs in an L1-heavy split would keep the attention CTAs (about
// 206 KB of shared memory each) that run beside it off those SMs.
template <typename K>
cudaError_t keep_smem_carveout(K kernel, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  if (done.load() & bit) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

// ---- TMA descriptor ----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D byte tensor [rows][inner] with row stride `stride` bytes; boxes of 128 bytes x 64
// rows, 128-byte swizzle.
ls_status make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LS_OK;
}

// 2D bf16 rows [rows][inner] (row stride in bytes), one-row boxes of 64 elements (128
// bytes), 128-byte swizzle: row gathers (tile::gather4) into K-major operand panels.
ls_status make_tmap_bf16_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
                              uint32_t box_rows = 1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed (%d)", (int)r);
  return LS_OK;
}

// ---- indexer launches ----------------------------------------------------------------
ls_status validate_index(const ls_index_score_args* a, bool need_scores) {
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->batch >= 1, "batch must be >= 1");
  LS_REQUIRE(a->max_pages >= 1 && a->max_len >= 1, "max_pages and max_len must be >= 1");
  LS_REQUIRE(a->num_pages >= 1, "num_pages must be >= 1");
  LS_REQUIRE(a->q && a->w && a->key_pool && a->page_table && a->lens, "a required pointer is NULL");
  LS_REQUIRE(!need_scores || a->scores, "scores is NULL");
  LS_REQUIRE(a->w_dtype == LS_BF16 || a->w_dtype == LS_F32, "w_dtype must be LS_BF16 or LS_F32");
  LS_REQUIRE(a->variant == 0 || a->variant == 1, "variant must be 0 or 1");
  if (a->key_dtype == LS_E4M3) {
    if (a->heads != 64 || a->dim != 128)
      return fail(LS_ERR_UNSUPPORTED, "e4m3 indexer is built for 64 heads x 128 dims (got %d x %d)", a->heads,
                  a->dim);
    LS_REQUIRE(a->q_scale && a->key_scale, "q_scale and key_scale are required for e4m3 keys");
    LS_REQUIRE(aligned16(a->q) && aligned16(a->key_pool) && aligned16(a->key_scale),
               "q, key_pool and key_scale must be 16-byte aligned");
  } else if (a->key_dtype == LS_F32) {
    if (a->heads < 1 || a->heads > 64 || a->dim < 1 || a->dim > 128 || (a->dim & 3))
      return fail(LS_ERR_UNSUPPORTED, "f32 indexer: heads in [1,64], dim in [4,128] multiple of 4");
    LS_REQUIRE(!a->q_scale && !a->key_scale, "q_scale/key_scale must be NULL for f32 keys");
  } else {
    return fail(LS_ERR_UNSUPPORTED, "key_dtype must be LS_E4M3 or LS_F32");
  }
  return LS_OK;
}

std::atomic<uint64_t> g_smem_idx_simt_f32{0}, g_smem_idx_simt_e4m3{0}, g_smem_idx_tc{0}, g_smem_idx_tc_f{0}, g_smem_bound_tc{0};

ls_status launch_index_simt(const ls_index_score_args* a, cudaStream_t st) {
  ls::IdxSimtParams p{};
  p.B = a->batch; p.H = a->heads; p.D = a->dim; p.max_pages = a->max_pages; p.max_len = a->max_len;
  p.num_pages = a->num_pages; p.q = a->q; p.qs = a->q_scale; p.w = a->w; p.w_bf16 = a->w_dtype == LS_BF16;
  p.keys = a->key_pool; p.ks = a->key_scale; p.page_table = a->page_table; p.lens = a->lens; p.out = a->scores;
  const int smem = (p.H * p.D + 64 * (p.D + 1) + p.H + 256) * 4;
  const int smem_max = (64 * 128 + 64 * 129 + 64 + 256) * 4;
  const int gx = std::min(a->max_pages, (a->max_len + 63) / 64);
  dim3 grid(gx, a->batch);
  if (a->key_dtype == LS_E4M3) {
    if (allow_smem(ls::index_score_simt<true>, smem_max, g_smem_idx_simt_e4m3) != cudaSuccess)
      return check_launch("index_score_simt attribute");
    ls::index_score_simt<true><<<grid, 256, smem, st>>>(p);
  } else {
    if (allow_smem(ls::index_score_simt<false>, smem_max, g_smem_idx_simt_f32) != cudaSuccess)
      return check_launch("index_score_simt attribute");
    ls::index_score_simt<false><<<grid, 256, smem, st>>>(p);
  }
  return check_launch("index_score_simt");
}

// tcgen05 tile engine over keys (mode 0) or block summaries (mode 1).
cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr,
                              bool pdl);

// CTAs per request of the tensor-core indexer: two (key scoring) or one (block bound) per SM
// over the batch, at most one per tile of two 64-row units.
int idx_ctas_per_req(int mode, int batch, long long max_units, int sms) {
  const long long max_tiles = (max_units + 1) / 2;
  const int per_sm = (mode == 0) ? 2 : 1;
  long long c = std::max<long long>(1, (long long)per_sm * sms / std::max(1, batch));
  return (int)std::min<long long>(c, std::max<long long>(1, max_tiles));
}

ls_status launch_index_tc(const ls_index_score_args* a, int mode, const int* unit_list, const int* unit_count,
                          int list_stride, float* out, long long out_stride, const uint8_t* summ,
                          const float* bscale, int max_blocks, float* out_plain, float eps_rel, cudaStream_t st,
                          int staged_base = -1, int stage_cap = 0, int* clear = nullptr,
                          const ls::IdxTcParams* filt = nullptr) {
  ls::IdxTcParams p{};
  p.clear = clear;
  if (filt) {  // the candidate filter's buffers
    p.filt = filt->filt;
    p.cand_cnt = filt->cand_cnt;
    p.cand_pos = filt->cand_pos;
    p.cand_score = filt->cand_score;
    p.filt_k = filt->filt_k;
  }
  p.staged = staged_base >= 0 ? 1 : 0;  // list entries [staged_base, + stage_cap) from staging units
  p.unit_base = staged_base >= 0 ? staged_base : 0;
  p.stage_cap = stage_cap;
  p.mode = mode; p.B = a->batch; p.max_pages = a->max_pages; p.max_len = a->max_len; p.max_blocks = max_blocks;
  p.num_pages = a->num_pages; p.q8 = (const uint8_t*)a->q; p.qs = a->q_scale; p.w = a->w;
  p.w_bf16 = a->w_dtype == LS_BF16; p.page_table = a->page_table; p.lens = a->lens;
  p.unit_list = unit_list; p.unit_count = unit_count; p.list_stride = list_stride;
  p.out = out; p.out_stride = out_stride; p.out_plain = out_plain; p.eps_rel = eps_rel;
  CUtensorMap tmap;
  const int sms = device_sms();
  long long max_units;
  if (mode == 0) {
    p.row_scale = a->key_scale;
    LS_TRY(make_tmap_u8(&tmap, a->key_pool, 128, (uint64_t)a->num_pages * 64, 128));
    max_units = unit_list ? (staged_base >= 0 ? std::min(list_stride, stage_cap) : list_stride)
                          : (a->max_len + 63) / 64;
  } else {
    p.row_scale = bscale;
    LS_TRY(make_tmap_u8(&tmap, summ, 256, (uint64_t)a->batch * max_blocks, 256));
    max_units = (max_blocks + 63) / 64;
  }
  const int c = idx_ctas_per_req(mode, a->batch, max_units, sms);
  p.ctas_per_req = c;
  dim3 grid((unsigned)c, a->batch);
  if (mode == 0) {
    if (p.filt) {  // the instance that keeps candidate lists
      using C = ls::IdxTc<1, 64, true>;
      if (allow_smem(ls::index_score_tc<1, 64, true>, C::kSmem, g_smem_idx_tc_f) != cudaSuccess)
        return check_launch("index_score_tc attribute");
      ls::index_score_tc<1, 64, true><<<grid, C::kThreads, C::kSmem, st>>>(p, tmap);
    } else {
      using C = ls::IdxTc<1, 64>;
      if (allow_smem(ls::index_score_tc<1, 64>, C::kSmem, g_smem_idx_tc) != cudaSuccess)
        return check_launch("index_score_tc attribute");
      ls::index_score_tc<1, 64><<<grid, C::kThreads, C::kSmem, st>>>(p, tmap);
    }
  } else {
    using C = ls::IdxTc<2, 128>;
    if (allow_smem(ls::index_score_tc<2, 128>, C::kSmem, g_smem_bound_tc) != cudaSuccess)
      return check_launch("block_bound_tc attribute");
    ls::index_score_tc<2, 128><<<grid, C::kThreads, C::kSmem, st>>>(p, tmap);
  }
  return check_launch(mode == 0 ? "index_score_tc" : "block_bound_tc");
}

// ---- top-k launch -------------------------------------------------------------------
// One cluster per request: 16 CTAs where the device can co-schedule them (non-portable
// cluster size), else the portable 8.
cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr,
                              bool pdl);
std::atomic<uint64_t> g_smem_topk8{0}, g_smem_topk16{0}, g_smem_topk_row{0};
// Requests up to this many candidates go to the one-CTA top-k, longer ones to a cluster
// (measured: at 131,072 scores per request one CTA takes ~50 us, a 16-CTA cluster ~20 us).
constexpr int kTopkRowMaxLen = 32768;
std::atomic<int> g_topk16_ok[kMaxDevices];  // per device: 0 unknown, 1 yes, -1 no

template <int CL>
cudaLaunchConfig_t topk_config(int B, int smem, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * CL);
  cfg.blockDim = dim3(ls::kTopkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // the kernel waits (griddepcontrol.wait) before reading anything, so it may always be
  // launched as a programmatic dependent of the kernel before
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

bool topk16_supported(cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return false;  // the 8-CTA launch then reports the ordinal
  std::atomic<int>& flag16 = g_topk16_ok[dev];
  int v = flag16.load();
  if (v != 0) return v > 0;
  bool ok = cudaFuncSetAttribute(ls::topk_cluster<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess;
  if (ok) ok = allow_smem(ls::topk_cluster<16>, ls::kTopkCacheKeys * 4 + ls::kTopkExtraBytes, g_smem_topk16) == cudaSuccess;
  if (ok) {
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = topk_config<16>(1, ls::kTopkCacheKeys * 4 + ls::kTopkExtraBytes, st, attr);
    int n = 0;
    ok = cudaOccupancyMaxActiveClusters(&n, ls::topk_cluster<16>, &cfg) == cudaSuccess && n >= 1;
  }
  cudaGetLastError();  // a refused probe leaves no sticky error
  flag16.store(ok ? 1 : -1);
  return ok;
}

template <int CL>
ls_status launch_topk_cl(const ls::TopkParams& p0, int B, cudaStream_t st, std::atomic<uint64_t>& smem_done) {
  ls::TopkParams p = p0;
  const int lc = (((p.len_limit + CL - 1) / CL) + 3) & ~3;
  p.cache_keys = lc <= ls::kTopkCacheKeys ? lc : 0;
  if (allow_smem(ls::topk_cluster<CL>, ls::kTopkCacheKeys * 4 + ls::kTopkExtraBytes, smem_done) != cudaSuccess)
    return check_launch("topk attribute");
  cudaLaunchAttribute attr[2];
  p.smem_bytes = p.cache_keys * 4 + ls::kTopkExtraBytes;
  cudaLaunchConfig_t cfg = topk_config<CL>(B, p.smem_bytes, st, attr);
  cudaError_t e = cudaLaunchKernelEx(&cfg, ls::topk_cluster<CL>, p);
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "topk_cluster: %s", cudaGetErrorString(e));
  return check_launch("topk_cluster");
}

ls_status launch_topk(int B, int k, const float* scores, int stride, const int* lens, int len_mul, int len_div,
                      int len_limit, const int* unit_list, int list_stride, int* idx, float* sel, float* thr,
                      cudaStream_t st, const int* pos_list = nullptr, int pos_stride = 0,
                      const int* pos_offset = nullptr, int* clear = nullptr, int* done = nullptr,
                      const ls::IdxTcParams* filt = nullptr, int filt_lists = 0,
                      const ls_sparse_attn_args* pf = nullptr) {
  ls::TopkParams p{};
  p.clear = clear;
  p.done = done;
  if (filt) {  // the indexer's candidate lists
    p.filt = filt->filt;
    p.cand_cnt = filt->cand_cnt;
    p.cand_pos = filt->cand_pos;
    p.cand_score = filt->cand_score;
    p.cand_lists = filt_lists;
    // the attention's bf16 paged rows, prefetched by the CTAs the candidate path leaves idle
    const bool pf_ok = pf && pf->addressing == LS_ROWS_PAGED && pf->dtype == LS_BF16 && pf->k_rows &&
                       pf->page_table && pf->row_stride >= pf->dk && pf->row_stride % 8 == 0 && pf->dk % 8 == 0 &&
                       ((uintptr_t)pf->k_rows & 15) == 0 && pf->num_rows > 0 && pf->max_pages > 0;
    if (pf_ok) {
      p.pf_rows = (const uint8_t*)pf->k_rows;
      p.pf_pt = pf->page_table;
      p.pf_max_pages = pf->max_pages;
      p.pf_num_rows = pf->num_rows;
      p.pf_row_bytes = pf->row_stride * 2;
      p.pf_bytes = pf->dk * 2;
    }
  }
  p.pos_list = pos_list; p.pos_stride = pos_stride; p.pos_offset = pos_offset;
  p.B = B; p.k = k; p.stride = stride; p.scores = scores; p.lens = lens; p.len_mul = len_mul;
  p.len_div = len_div; p.len_limit = len_limit; p.unit_list = unit_list; p.list_stride = list_stride;
  p.idx = idx; p.sel = sel; p.thr = thr;
  if (len_limit <= kTopkRowMaxLen) {
    // one CTA per request: few SMs for a small batch and no cluster barriers
    if (allow_smem(ls::topk_row, ls::kRowSmem, g_smem_topk_row) != cudaSuccess)
      return check_launch("topk_row attribute");
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pdl_config(dim3(B), dim3(ls::kRowThreads), ls::kRowSmem, st, attr, true);
    cudaError_t e = cudaLaunchKernelEx(&cfg, ls::topk_row, p);
    if (e != cudaSuccess) return fail(LS_ERR_CUDA, "topk_row: %s", cudaGetErrorString(e));
    return check_launch("topk_row");
  }
  if (topk16_supported(st)) return launch_topk_cl<16>(p, B, st, g_smem_topk16);
  return launch_topk_cl<8>(p, B, st, g_smem_topk8);
}

// ---- attention ------------------------------------------------------------------------
int attn_nsplit(const ls_sparse_attn_args* a) {
  if (a->dtype != LS_BF16 || a->variant != 0) return 1;
  const int tiles = (a->k + ls::mla::N - 1) / ls::mla::N;
  int ns = device_sms() / (2 * a->batch);
  ns = std::max(1, std::min(ns, (tiles + 1) / 2));
  // the fewest splits with the same longest share (e.g. 32 tiles: 8 splits of 4, not 9 of
  // 3-4): the same critical path, fewer partials to store and merge, SMs left free
  const int per = (tiles + ns - 1) / ns;
  return (tiles + per - 1) / per;
}

std::atomic<uint64_t> g_smem_attn_tc{0}, g_smem_attn_simt_f{0}, g_smem_attn_simt_b{0};

// Most clusters of 2 * ns tensor-core attention CTAs the device runs at once (asked once
// per device and split count); 0 when such a cluster cannot be launched.
int attn_max_clusters(int ns) {
  static std::atomic<int> cache[kMaxDevices][ls::mla::kMergeBatch + 1];  // 0 unknown, -1 none
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices || ns < 1 || ns > ls::mla::kMergeBatch) return 0;
  const int known = cache[dev][ns].load();
  if (known != 0) return known > 0 ? known : 0;
  int n = 0;
  bool ok = allow_smem(ls::attn_mla_tc, ls::mla::kSmem, g_smem_attn_tc) == cudaSuccess;
  if (ok && 2 * ns > 8)
    ok = cudaFuncSetAttribute(ls::attn_mla_tc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(2 * ns, 1);
    cfg.blockDim = dim3(ls::mla::kThreads);
    cfg.dynamicSmemBytes = ls::mla::kSmem;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2 * ns;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ok = cudaOccupancyMaxActiveClusters(&n, ls::attn_mla_tc, &cfg) == cudaSuccess && n > 0;
  }
  cudaGetLastError();  // a refused query leaves no sticky error
  cache[dev][ns].store(ok ? n : -1);
  return ok ? n : 0;
}

// Whether the splits of a tensor-core attention launch are merged inside one cluster per
// request instead of by attn_combine: one pass, a bf16 output, a split count that divides
// the heads (2, 4 or 8 -- at most a 16-CTA cluster), and every request's cluster resident
// at once (otherwise the clusters would run in waves).
bool attn_merge(const ls_sparse_attn_args* a, int npasses) {
  if (a->dtype != LS_BF16 || a->variant != 0 || npasses != 1 || a->o_f32) return false;
  const int ns = attn_nsplit(a);
  if (ns != 2 && ns != 4 && ns != 8) return false;
  return attn_max_clusters(ns) >= a->batch;
}

// Split-KV partials of `npasses` launches over the same requests (each with
// attn_nsplit splits), merged by one combine; none when the splits merge in the cluster.
size_t attn_ws_bytes(const ls_sparse_attn_args* a, int npasses = 1) {
  const int ns = attn_nsplit(a) * npasses;
  if (ns <= 1 || attn_merge(a, npasses)) return 0;
  return align256((size_t)a->batch * ns * a->heads * a->dv * 4) + align256((size_t)a->batch * ns * a->heads * 8);
}

ls_status validate_attn(const ls_sparse_attn_args* a, bool need_sel) {
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->batch >= 1 && a->k >= 1 && a->k <= 4096, "batch >= 1 and 1 <= k <= 4096 required");
  LS_REQUIRE(a->q && a->k_rows && a->v_rows && a->o && a->lse, "a required pointer is NULL");
  LS_REQUIRE(!need_sel || a->sel, "sel is NULL");
  LS_REQUIRE(a->addressing == LS_ROWS_PAGED || a->addressing == LS_ROWS_SLOTS, "bad addressing mode");
  LS_REQUIRE(a->addressing != LS_ROWS_PAGED || (a->page_table && a->max_pages >= 1),
             "paged addressing needs page_table and max_pages");
  LS_REQUIRE(a->addressing != LS_ROWS_SLOTS || a->n_slots >= 1, "slot addressing needs n_slots");
  LS_REQUIRE(a->num_rows >= 1, "num_rows must be >= 1");
  LS_REQUIRE(a->variant == 0 || a->variant == 1, "variant must be 0 or 1");
  LS_REQUIRE(std::isfinite(a->softmax_scale), "softmax_scale must be finite");
  if (a->dtype == LS_BF16) {
    if (a->variant == 0 && (a->heads != 128 || a->dk != 576 || a->dv != 512))
      return fail(LS_ERR_UNSUPPORTED, "bf16 tensor-core attention is built for 128 heads, dk 576, dv 512");
    if (a->variant == 0) {
      LS_REQUIRE(aligned16(a->o), "o must be 16-byte aligned");
      LS_REQUIRE(a->k_rows == a->v_rows, "MLA attention reads V from the latent rows (v_rows == k_rows)");
      LS_REQUIRE(a->row_stride >= 576 && (a->row_stride % 8) == 0, "row_stride must be >= 576 and % 8 == 0");
      LS_REQUIRE(a->num_rows < 0x7fffffffLL, "num_rows must be below 2^31 - 1");
      LS_REQUIRE(aligned16(a->k_rows) && aligned16(a->q), "k_rows and q must be 16-byte aligned");
    }
  } else if (a->dtype != LS_F32) {
    return fail(LS_ERR_UNSUPPORTED, "attention dtype must be LS_BF16 or LS_F32");
  }
  if ((a->variant == 1 && a->dtype == LS_BF16) && a->o_f32)
    return fail(LS_ERR_UNSUPPORTED, "o_f32 is built for the tensor-core bf16 kernel (variant 0)");
  if (a->variant == 1 || a->dtype == LS_F32) {
    LS_REQUIRE(a->heads >= 1 && a->dk >= 1 && a->dv >= 1 && a->dk <= 1024 && a->dv <= 1024,
               "CUDA-core attention: heads >= 1, 1 <= dk, dv <= 1024");
    LS_REQUIRE(a->row_stride >= std::max(a->dk, a->dv), "row_stride must cover dk and dv");
  }
  return LS_OK;
}

// Programmatic dependent launch: the kernel may start while the one before it finishes
// (it waits for it with griddepcontrol.wait before touching its output).
cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr,
                              bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cfg;
}

// `pdl`: launched right behind another kernel of the same decode step, whose outputs
// (selection, or gathered rows) the attention reads; Q is not among them.  `compacted`:
// every request's valid selection entries come first.  Pass `pass` of `npasses`
// (tensor-core path): the launch fills its own range of split-KV partials; `combine`
// merges all passes' partials into o and lse.
ls_status launch_attn(const ls_sparse_attn_args* a, const int* sel, int addressing, const int* page_table,
                      int max_pages, int n_slots, const void* rows, long long num_rows, void* ws, size_t ws_bytes,
                      cudaStream_t st, bool pdl, bool compacted = false, int pass = 0, int npasses = 1,
                      bool combine = true, const int* n_valid = nullptr, int* done = nullptr,
                      const int* ready = nullptr, int ready_want = 0) {
  ls::AttnParams p{};
  p.B = a->batch; p.H = a->heads; p.dk = a->dk; p.dv = a->dv; p.k = a->k; p.scale = a->softmax_scale;
  p.addressing = addressing; p.max_pages = max_pages; p.n_slots = n_slots; p.row_stride = a->row_stride;
  p.num_rows = num_rows; p.q = a->q; p.krows = rows ? rows : a->k_rows; p.vrows = rows ? rows : a->v_rows;
  p.page_table = page_table; p.sel = sel; p.o = a->o; p.lse = a->lse;
  if (a->dtype == LS_BF16 && a->variant == 0) {
    const int ns = attn_nsplit(a);
    const int total = ns * npasses;
    p.nsplit = ns;
    p.split_base = pass * ns;
    p.nsplit_total = total;
    p.compacted = compacted ? 1 : 0;
    p.o_f32 = a->o_f32 ? 1 : 0;
    p.n_valid = n_valid;
    const bool merge = attn_merge(a, npasses);
    p.merge = merge ? 1 : 0;
    // a per-request completion count lets the combine start request by request; only for a
    // single pass whose count the kernel before (the top-k) has just zeroed
    p.done = (total > 1 && !merge && combine && npasses == 1) ? done : nullptr;
    p.ready = ready;
    p.ready_want = ready_want;
    if (total > 1 && !merge) {
      const size_t need = attn_ws_bytes(a, npasses);
      LS_REQUIRE(ws && ws_bytes >= need, "attention workspace too small (%zu < %zu bytes)", ws_bytes, need);
      LS_REQUIRE(((uintptr_t)ws & 255) == 0, "workspace must be 256-byte aligned");
      p.part_o = (float*)ws;
      p.part_ml = (float*)((char*)ws + align256((size_t)a->batch * total * a->heads * a->dv * 4));
    }
    if (allow_smem(ls::attn_mla_tc, ls::mla::kSmem, g_smem_attn_tc) != cudaSuccess)
      return check_launch("attn_mla_tc attribute");
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pdl_config(dim3(2 * ns, a->batch), dim3(ls::mla::kThreads), ls::mla::kSmem, st, attr, pdl);
    // the two CTAs of an (request, split) pair form a cluster; with the in-cluster merge,
    // all splits of a request do
    attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
    attr[cfg.numAttrs].val.clusterDim.x = merge ? 2 * ns : 2;
    attr[cfg.numAttrs].val.clusterDim.y = 1;
    attr[cfg.numAttrs].val.clusterDim.z = 1;
    cfg.numAttrs += 1;
    CUtensorMap kv_map;
    LS_TRY(make_tmap_bf16_rows(&kv_map, p.krows, ls::mla::DK, (uint64_t)num_rows, (uint64_t)a->row_stride * 2));
    CUtensorMap q_map;  // [B*128 heads, 576] bf16, one 128-head x 64-dim box per panel
    LS_TRY(make_tmap_bf16_rows(&q_map, p.q, ls::mla::DK, (uint64_t)a->batch * ls::mla::H, ls::mla::DK * 2,
                               ls::mla::H));
    cudaError_t e = cudaLaunchKernelEx(&cfg, ls::attn_mla_tc, p, kv_map, q_map);
    if (e != cudaSuccess) return fail(LS_ERR_CUDA, "attn_mla_tc: %s", cudaGetErrorString(e));
    LS_TRY(check_launch("attn_mla_tc"));
    if (total > 1 && combine && !merge) {
      cudaLaunchConfig_t cc = pdl_config(dim3(ls::mla::H * ls::mla::DV / 8 / ls::kCombineThreads, a->batch),
                                         dim3(ls::kCombineThreads), 0, st, attr, true);
      e = cudaLaunchKernelEx(&cc, ls::attn_combine, p);
      if (e != cudaSuccess) return fail(LS_ERR_CUDA, "attn_combine: %s", cudaGetErrorString(e));
      LS_TRY(check_launch("attn_combine"));
    }
    return LS_OK;
  }
  const int smem = (((a->dk + 1) & ~1) + ((a->k + 1) & ~1)) * 4 + a->k * 8;
  LS_REQUIRE(smem <= 200 * 1024, "CUDA-core attention: dk + 3k too large for shared memory");
  dim3 grid(a->heads, a->batch);
  if (a->dtype == LS_BF16) {
    if (allow_smem(ls::attn_simt<true>, 200 * 1024, g_smem_attn_simt_b) != cudaSuccess)
      return check_launch("attn_simt attribute");
    ls::attn_simt<true><<<grid, 256, smem, st>>>(p);
  } else {
    if (allow_smem(ls::attn_simt<false>, 200 * 1024, g_smem_attn_simt_f) != cudaSuccess)
      return check_launch("attn_simt attribute");
    ls::attn_simt<false><<<grid, 256, smem, st>>>(p);
  }
  return check_launch("attn_simt");
}

// ---- hot buffer -------------------------------------------------------------------------
std::atomic<uint64_t> g_smem_hb{0}, g_carve_hb{0}, g_carve_gather{0}, g_carve_classify{0}, g_carve_copy{0};

ls_status validate_hotbuf(const ls_hotbuf_args* a) {
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->batch >= 1 && a->k >= 1, "batch and k must be >= 1");
  LS_REQUIRE(a->n_slots >= 1 && a->n_slots <= ls::kHbMaxSlots, "n_slots must be in [1, 4096]");
  LS_REQUIRE(a->k <= a->n_slots, "k must not exceed n_slots (every selection needs a slot)");
  LS_REQUIRE(a->max_len >= 1, "max_len must be >= 1");
  LS_REQUIRE(a->sel && a->sel_score && a->pos_of_slot && a->recent_score && a->slot_of_pos && a->sel_slot &&
                 a->miss_pos && a->miss_slot && a->n_miss,
             "a required pointer is NULL");
  return LS_OK;
}

ls_status launch_hotbuf(const ls_hotbuf_args* a, cudaStream_t st) {
  ls::HotbufParams p{};
  p.B = a->batch; p.k = a->k; p.n_slots = a->n_slots; p.max_len = a->max_len; p.sel = a->sel;
  p.sel_score = a->sel_score; p.pos_of_slot = a->pos_of_slot; p.recent = a->recent_score;
  p.slot_of_pos = a->slot_of_pos; p.sel_slot = a->sel_slot; p.miss_pos = a->miss_pos; p.miss_slot = a->miss_slot;
  p.n_miss = a->n_miss;
  if (allow_smem(ls::hotbuf_resolve_kernel, ls::kHbResolveSmem, g_smem_hb) != cudaSuccess ||
      keep_smem_carveout(ls::hotbuf_resolve_kernel, g_carve_hb) != cudaSuccess)
    return check_launch("hotbuf attribute");
  ls::hotbuf_resolve_kernel<<<a->batch, ls::kHbThreads, ls::kHbResolveSmem, st>>>(p);
  return check_launch("hotbuf_resolve");
}

ls_status validate_gather(const ls_gather_args* a) {
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->batch >= 1 && a->k >= 1 && a->n_slots >= 1 && a->max_pages >= 1 && a->num_pages >= 1,
             "batch, k, n_slots, max_pages, num_pages must be >= 1");
  LS_REQUIRE(a->row_bytes >= 16 && (a->row_bytes % 16) == 0, "row_bytes must be a positive multiple of 16");
  LS_REQUIRE(a->host_kv && a->page_table && a->miss_pos && a->miss_slot && a->n_miss && a->hbuf,
             "a required pointer is NULL");
  LS_REQUIRE(aligned16(a->host_kv) && aligned16(a->hbuf), "host_kv and hbuf must be 16-byte aligned");
  return LS_OK;
}

ls_status launch_gather(const ls_gather_args* a, cudaStream_t st, void* stage = nullptr) {
  ls::GatherParams p{};
  p.B = a->batch; p.k = a->k; p.n_slots = a->n_slots; p.max_pages = a->max_pages; p.row_bytes = a->row_bytes;
  p.num_pages = a->num_pages; p.host = (const char*)a->host_kv; p.page_table = a->page_table;
  p.miss_pos = a->miss_pos; p.miss_slot = a->miss_slot; p.n_miss = a->n_miss; p.hbuf = (char*)a->hbuf;
  p.stage = (char*)stage;
  // small CTAs on about a quarter of the SMs: 144 warps with two rows each in flight keep
  // the host link busy (measured: as fast as one CTA per SM), and the attention on the
  // resident rows, which runs beside the gather in the decode step, is slowed far less
  // by a gather CTA on its SM
  const int rows_per_cta = (ls::kGatherThreads / 32) * 2;
  int g = (a->k + rows_per_cta - 1) / rows_per_cta;
  g = std::max(1, std::min(g, device_sms() / (4 * a->batch)));
  if (keep_smem_carveout(ls::gather_misses_kernel, g_carve_gather) != cudaSuccess)
    return check_launch("gather attribute");
  ls::gather_misses_kernel<<<dim3(g, a->batch), ls::kGatherThreads, 0, st>>>(p);
  return check_launch("gather_misses");
}

// The decode step's classification of the selection (resident slots; misses compacted
// in selection order) ahead of the full resolve.
ls_status launch_classify(const ls_hotbuf_args* a, int* hit_slot, int* n_hit, int* miss_pos, int* miss_row,
                          int* n_miss, cudaStream_t st) {
  ls::ClassifyParams p{};
  p.B = a->batch; p.k = a->k; p.n_slots = a->n_slots; p.max_len = a->max_len; p.sel = a->sel;
  p.slot_of_pos = a->slot_of_pos; p.hit_slot = hit_slot; p.n_hit = n_hit; p.miss_pos = miss_pos; p.miss_row = miss_row;
  p.n_miss = n_miss;
  if (keep_smem_carveout(ls::hotbuf_classify_kernel, g_carve_classify) != cudaSuccess)
    return check_launch("classify attribute");
  ls::hotbuf_classify_kernel<<<a->batch, ls::kHbThreads, 0, st>>>(p);
  return check_launch("hotbuf_classify");
}

// Staged miss rows into the victim slots the resolve chose.
ls_status launch_copy_staged(const ls_gather_args* g, const void* stage, cudaStream_t st) {
  ls::StageCopyParams p{};
  p.B = g->batch; p.k = g->k; p.n_slots = g->n_slots; p.row_bytes = g->row_bytes; p.stage = (const char*)stage;
  p.miss_slot = g->miss_slot; p.n_miss = g->n_miss; p.hbuf = (char*)g->hbuf;
  int c = (g->k + 7) / 8;
  c = std::max(1, std::min(c, (4 * device_sms()) / g->batch + 1));
  if (keep_smem_carveout(ls::copy_staged_kernel, g_carve_copy) != cudaSuccess)
    return check_launch("copy_staged attribute");
  ls::copy_staged_kernel<<<dim3(c, g->batch), 256, 0, st>>>(p);
  return check_launch("copy_staged");
}

// ---- coarse-to-fine ---------------------------------------------------------------------
struct C2fLayout {
  int nb0, ub_stride, cap;
  size_t off_ub, off_blk, off_cnt1, off_clen1, off_tau, off_clen2, off_nsurv, off_surv, off_c1, off_c2, off_skeys,
      off_sscales, total;
};

C2fLayout c2f_layout(const ls_block_bound_prune_args* a) {
  C2fLayout l{};
  const int B = a->index.batch;
  l.nb0 = std::min(a->max_blocks, (a->k + 63) / 64 + 1);
  l.ub_stride = (a->max_blocks + 3) & ~3;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += align256(bytes); return r; };
  l.off_ub = take((size_t)B * l.ub_stride * 4);
  l.off_blk = take((size_t)B * l.nb0 * 4);
  l.off_cnt1 = take((size_t)B * 4);
  l.off_clen1 = take((size_t)B * 4);
  l.off_tau = take((size_t)B * 4);
  l.off_clen2 = take((size_t)B * 4);
  l.off_nsurv = take((size_t)B * 4);
  l.off_surv = take((size_t)B * a->max_blocks * 4);
  l.off_c1 = take((size_t)B * l.nb0 * 64 * 4);
  l.off_c2 = take((size_t)B * a->max_blocks * 64 * 4);
  l.cap = 0;
  if (a->keys_on_host) {  // staging for the keys fetched from the host, per pass
    l.cap = std::min(a->max_blocks, std::max(l.nb0, a->stage_blocks > 0 ? a->stage_blocks : 2048));
    l.off_skeys = take((size_t)B * l.cap * 8192);
    l.off_sscales = take((size_t)B * l.cap * 256);
  }
  l.total = o;
  return l;
}

ls_status validate_c2f(const ls_block_bound_prune_args* a) {
  LS_REQUIRE(a, "args is NULL");
  LS_TRY(validate_index(&a->index, false));
  if (a->index.key_dtype != LS_E4M3) return fail(LS_ERR_UNSUPPORTED, "coarse-to-fine needs e4m3 indexer keys");
  LS_REQUIRE(a->k >= 1 && a->k <= 4096, "1 <= k <= 4096 required");
  LS_REQUIRE(a->max_blocks >= 1, "max_blocks must be >= 1");
  LS_REQUIRE((long long)a->max_blocks * 64 <= (1ll << 30), "max_blocks too large");
  LS_REQUIRE(a->summaries && a->block_scale && a->idx, "summaries, block_scale and idx are required");
  LS_REQUIRE(aligned16(a->summaries), "summaries must be 16-byte aligned");
  LS_REQUIRE(a->stage_blocks >= 0, "stage_blocks must be >= 0");
  return LS_OK;
}

// Device addresses of host-resident keys and scales: both must be pinned host memory.
ls_status host_key_ptrs(const ls_index_score_args* ix, const uint8_t** keys, const float** scales) {
  const void* src[2] = {ix->key_pool, ix->key_scale};
  void* dev[2] = {nullptr, nullptr};
  for (int i = 0; i < 2; ++i) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, src[i]) != cudaSuccess || at.type != cudaMemoryTypeHost || !at.devicePointer) {
      cudaGetLastError();
      return fail(LS_ERR_INVALID_ARG, "keys_on_host: index.%s is not pinned host memory",
                  i == 0 ? "key_pool" : "key_scale");
    }
    dev[i] = at.devicePointer;
  }
  *keys = (const uint8_t*)dev[0];
  *scales = (const float*)dev[1];
  return LS_OK;
}

// List entries [base, base + cap) of each request: their keys over the host link into
// staging, then their exact scores into out (at the entries' own positions).
ls_status fetch_and_score(const ls_index_score_args* ix, const uint8_t* hkeys, const float* hscales,
                          const int* list, const int* count, int list_stride, int base, int cap, uint8_t* skeys,
                          float* sscales, float* out, long long out_stride, cudaStream_t st) {
  ls::FetchParams f{};
  f.B = ix->batch; f.max_pages = ix->max_pages; f.list_stride = list_stride; f.base = base; f.cap = cap;
  f.num_pages = ix->num_pages; f.host_keys = hkeys; f.host_scales = hscales; f.page_table = ix->page_table;
  f.list = list; f.count = count; f.stage_keys = skeys; f.stage_scales = sscales;
  // small CTAs on about a quarter of the SMs keep enough loads in flight for the link
  const int g = std::max(1, std::min((cap + 3) / 4, device_sms() / (4 * ix->batch)));
  ls::fetch_blocks_kernel<<<dim3(g, ix->batch), 128, 0, st>>>(f);
  LS_TRY(check_launch("fetch_blocks"));
  ls_index_score_args tmp = *ix;
  tmp.key_pool = skeys;
  tmp.key_scale = sscales;
  tmp.num_pages = (int64_t)ix->batch * cap;
  return launch_index_tc(&tmp, 0, list, count, list_stride, out, out_stride, nullptr, nullptr, 0, nullptr, 0.f, st,
                         base, cap);
}

ls_status run_c2f(const ls_block_bound_prune_args* a, void* ws, size_t ws_bytes, int* survivors, int* n_surv,
                  ls_event_t ev_topk, cudaStream_t st) {
  const C2fLayout l = c2f_layout(a);
  LS_REQUIRE(ws && ws_bytes >= l.total, "coarse-to-fine workspace too small (%zu < %zu bytes)", ws_bytes, l.total);
  LS_REQUIRE(((uintptr_t)ws & 255) == 0, "workspace must be 256-byte aligned");
  char* w = (char*)ws;
  float* ub = (float*)(w + l.off_ub);
  int* blk = (int*)(w + l.off_blk);
  int* cnt1 = (int*)(w + l.off_cnt1);
  int* clen1 = (int*)(w + l.off_clen1);
  float* tau = (float*)(w + l.off_tau);
  int* clen2 = (int*)(w + l.off_clen2);
  if (!n_surv) n_surv = (int*)(w + l.off_nsurv);
  if (!survivors) survivors = (int*)(w + l.off_surv);
  float* c1 = (float*)(w + l.off_c1);
  float* c2 = (float*)(w + l.off_c2);
  const ls_index_score_args* ix = &a->index;
  const int B = ix->batch;
  const float eps = a->eps_rel > 0.f ? a->eps_rel : 1.0f / 1024.0f;
  const uint8_t* hkeys = nullptr;
  const float* hscales = nullptr;
  uint8_t* skeys = (uint8_t*)(w + l.off_skeys);
  float* sscales = (float*)(w + l.off_sscales);
  if (a->keys_on_host) LS_TRY(host_key_ptrs(ix, &hkeys, &hscales));
  // 1. block bounds (+ margin) over the summaries
  LS_TRY(launch_index_tc(ix, 1, nullptr, nullptr, 0, ub, l.ub_stride, a->summaries, a->block_scale, a->max_blocks,
                         a->ub, eps, st));
  // 2. the blocks with the largest bounds
  LS_TRY(launch_topk(B, l.nb0, ub, l.ub_stride, ix->lens, 1, 64, a->max_blocks, nullptr, 0, blk, nullptr, nullptr,
                     st));
  ls::c2f_phase1_kernel<<<(B + 127) / 128, 128, 0, st>>>(B, l.nb0, ix->lens, blk, cnt1, clen1);
  LS_TRY(check_launch("c2f_phase1"));
  // 3. their exact scores; tau0 = the k-th largest
  if (a->keys_on_host) {
    LS_TRY(fetch_and_score(ix, hkeys, hscales, blk, cnt1, l.nb0, 0, l.cap, skeys, sscales, c1, (long long)l.nb0 * 64,
                           st));
  } else {
    LS_TRY(launch_index_tc(ix, 0, blk, cnt1, l.nb0, c1, (long long)l.nb0 * 64, nullptr, nullptr, 0, nullptr, 0.f,
                           st));
  }
  LS_TRY(launch_topk(B, a->k, c1, l.nb0 * 64, clen1, 1, 1, l.nb0 * 64, nullptr, 0, nullptr, nullptr, tau, st));
  // 4. survivors
  ls::c2f_survivors_kernel<<<B, 1024, 0, st>>>(B, a->max_blocks, l.ub_stride, ix->lens, ub, tau, survivors, n_surv,
                                               clen2);
  LS_TRY(check_launch("c2f_survivors"));
  // 5. exact scores of the survivors, then the top-k over them
  if (a->keys_on_host) {
    // the survivors through the staging, stage-capacity blocks per pass (a pass past a
    // request's survivor count does nothing for it)
    for (int base = 0; base < a->max_blocks; base += l.cap)
      LS_TRY(fetch_and_score(ix, hkeys, hscales, survivors, n_surv, a->max_blocks, base, l.cap, skeys, sscales, c2,
                             (long long)a->max_blocks * 64, st));
  } else {
    LS_TRY(launch_index_tc(ix, 0, survivors, n_surv, a->max_blocks, c2, (long long)a->max_blocks * 64, nullptr,
                           nullptr, 0, nullptr, 0.f, st));
  }
  if (ev_topk) cudaEventRecord((cudaEvent_t)ev_topk, st);
  LS_TRY(launch_topk(B, a->k, c2, a->max_blocks * 64, clen2, 1, 1, a->max_blocks * 64, survivors, a->max_blocks,
                     a->idx, a->sel_score, nullptr, st));
  return LS_OK;
}

// ---- decode step workspace ------------------------------------------------------------
struct StepLayout {
  size_t off_scores, off_idx, off_sel, off_selslot, off_mpos, off_mslot, off_nmiss, off_hitslot, off_cpos, off_crow,
      off_cnmiss, off_cnhit, off_stage, off_attn, off_done, off_ready, off_filt, off_candcnt, off_candpos,
      off_candscore, off_c2f, total;
};

ls_block_bound_prune_args step_c2f_args(const ls_decode_step_args* a, int* idx, float* sel) {
  ls_block_bound_prune_args c{};
  c.index = a->index;
  c.k = a->k;
  c.max_blocks = a->max_blocks;
  c.eps_rel = a->eps_rel;
  c.summaries = a->summaries;
  c.block_scale = a->block_scale;
  c.idx = idx;
  c.sel_score = sel;
  c.survivors = a->survivors;
  c.n_survivors = a->n_survivors;
  c.ub = nullptr;
  c.keys_on_host = a->c2f_keys_on_host;
  c.stage_blocks = a->c2f_stage_blocks;
  return c;
}

// Merge the split-KV partials of `npasses` tensor-core attention launches into o and lse.
ls_status launch_attn_combine(const ls_sparse_attn_args* a, void* ws, int npasses, cudaStream_t st) {
  ls::AttnParams p{};
  p.B = a->batch; p.H = a->heads; p.dk = a->dk; p.dv = a->dv; p.k = a->k; p.o = a->o; p.lse = a->lse;
  p.o_f32 = a->o_f32 ? 1 : 0;
  const int ns = attn_nsplit(a), total = ns * npasses;
  p.nsplit = ns;
  p.nsplit_total = total;
  p.part_o = (float*)ws;
  p.part_ml = (float*)((char*)ws + align256((size_t)a->batch * total * a->heads * a->dv * 4));
  ls::attn_combine<<<dim3(ls::mla::H * ls::mla::DV / 8 / ls::kCombineThreads, a->batch), ls::kCombineThreads, 0,
                     st>>>(p);
  return check_launch("attn_combine");
}

// Whether the hot-buffer step attends to the resident rows while the misses are being
// gathered (tensor-core attention), or strictly after the gather.
bool overlap_misses(const ls_sparse_attn_args* at) { return at->dtype == LS_BF16 && at->variant == 0; }

// Two more streams of this host thread for one (device, caller stream), and the events for
// the fork and joins of the overlapped hot-buffer step (created once, reused).  Keyed by the
// caller's stream, so that steps issued from one thread on independent streams neither
// share side streams (a false serialisation) nor re-record each other's events (a join on
// the wrong step); calls on one stream are ordered, so their reuse is safe.
struct SideStream {
  cudaStream_t s[2] = {nullptr, nullptr};
  cudaEvent_t fork = nullptr, gathered = nullptr, join[2] = {nullptr, nullptr};
};
ls_status side_stream(cudaStream_t caller, SideStream** out) {
  thread_local std::map<std::pair<int, cudaStream_t>, SideStream> per_stream;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return fail(LS_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  SideStream& ss = per_stream[std::make_pair(dev, caller)];
  if (!ss.s[1]) {
    bool good = true;
    for (int i = 0; i < 2; ++i) {
      if (!ss.s[i]) good = good && cudaStreamCreateWithFlags(&ss.s[i], cudaStreamNonBlocking) == cudaSuccess;
      if (!ss.join[i]) good = good && cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming) == cudaSuccess;
    }
    if (!ss.fork) good = good && cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess;
    if (!ss.gathered) good = good && cudaEventCreateWithFlags(&ss.gathered, cudaEventDisableTiming) == cudaSuccess;
    if (!good) {
      ss.s[1] = nullptr;
      return check_launch("side streams");
    }
  }
  *out = &ss;
  return LS_OK;
}

ls_sparse_attn_args step_attn_args(const ls_decode_step_args* a) {
  ls_sparse_attn_args t = a->attn;
  t.batch = a->index.batch;
  t.k = a->k;
  return t;
}

// The indexer's CTAs per request in the decode step (the layout of the candidate lists).
int step_idx_ctas(const ls_decode_step_args* a);

// Whether the step's indexer keeps candidate lists for the cluster top-k: the tensor-core
// indexer over whole requests (not the coarse-to-fine pass), requests long enough for the
// cluster top-k and short enough for its key cache (the candidate path's position bitmap
// shares that room), k within the candidates the path holds, and enough tiles per indexer CTA
// (at least 12) for the threshold to arrive while a CTA still has tiles to score.
bool step_uses_candidates(const ls_decode_step_args* a) {
  const ls_index_score_args* ix = &a->index;
  if (a->use_c2f || ix->key_dtype != LS_E4M3 || ix->variant != 0 || ix->max_len <= kTopkRowMaxLen ||
      ix->max_len > 16 * ls::kTopkCacheKeys || a->k < 1 || a->k > ls::kFastMaxCand)
    return false;
  const long long tiles = (((long long)ix->max_len + 63) / 64 + 1) / 2;
  return tiles >= 12LL * step_idx_ctas(a);
}

// The indexer's CTAs per request in the decode step (the layout of the candidate lists).
int step_idx_ctas(const ls_decode_step_args* a) {
  return idx_ctas_per_req(0, a->index.batch, ((long long)a->index.max_len + 63) / 64, device_sms());
}

StepLayout step_layout(const ls_decode_step_args* a) {
  StepLayout l{};
  const int B = a->index.batch, k = a->k;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += align256(bytes); return r; };
  l.off_scores = take(a->use_c2f ? 0 : (size_t)B * a->index.max_len * 4);
  l.off_idx = take((size_t)B * k * 4);
  l.off_sel = take((size_t)B * k * 4);
  l.off_selslot = take(a->use_hotbuf ? (size_t)B * k * 4 : 0);
  l.off_mpos = take(a->use_hotbuf ? (size_t)B * k * 4 : 0);
  l.off_mslot = take(a->use_hotbuf ? (size_t)B * k * 4 : 0);
  l.off_nmiss = take(a->use_hotbuf ? (size_t)B * 4 : 0);
  ls_sparse_attn_args t = step_attn_args(a);
  const bool two_pass = a->use_hotbuf && overlap_misses(&t);
  l.off_hitslot = take(two_pass ? (size_t)B * k * 4 : 0);
  l.off_cpos = take(two_pass ? (size_t)B * k * 4 : 0);
  l.off_crow = take(two_pass ? (size_t)B * k * 4 : 0);
  l.off_cnmiss = take(two_pass ? (size_t)B * 4 : 0);
  l.off_cnhit = take(two_pass ? (size_t)B * 4 : 0);
  l.off_stage = take(two_pass ? (size_t)B * k * t.row_stride * 2 : 0);
  l.off_attn = take(attn_ws_bytes(&t, two_pass ? 2 : 1));
  l.off_done = take((size_t)B * 4);   // per-request attention completion counts
  l.off_ready = take((size_t)B * 4);  // per-request top-k completion counts
  // the indexer's candidate filter and the candidate top-k (whole requests of the paged or
  // hot-buffer step whose top-k is the cluster kernel)
  const bool cand = step_uses_candidates(a);
  const size_t cpr = cand ? (size_t)step_idx_ctas(a) : 0;
  l.off_filt = take(cand ? (size_t)B * ls::kFiltInts * 4 : 0);
  l.off_candcnt = take((size_t)B * cpr * 4 * 4);
  l.off_candpos = take((size_t)B * cpr * ls::kCandPerCta * 4);
  l.off_candscore = take((size_t)B * cpr * ls::kCandPerCta * 4);
  if (a->use_c2f) {
    ls_block_bound_prune_args c = step_c2f_args(a, nullptr, nullptr);
    l.off_c2f = take(c2f_layout(&c).total);
  } else {
    l.off_c2f = o;
  }
  l.total = o;
  return l;
}

// ---- layer-streaming prefill --------------------------------------------------------
struct PrefillLayout {
  size_t off_keys[2], off_scales[2], off_spos, off_sslot, off_sn, total;
};

PrefillLayout prefill_layout(const ls_prefill_stream_args* a) {
  PrefillLayout l{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += align256(bytes); return r; };
  for (int i = 0; i < 2; ++i) {
    l.off_keys[i] = take((size_t)a->num_pages * 64 * 128);
    l.off_scales[i] = take((size_t)a->num_pages * 64 * 4);
  }
  const size_t ns = a->n_slots > 0 ? (size_t)a->batch * a->n_slots * 4 : 0;
  l.off_spos = take(ns);
  l.off_sslot = take(ns);
  l.off_sn = take(a->n_slots > 0 ? (size_t)a->batch * 4 : 0);
  l.total = o;
  return l;
}

bool pinned_host(const void* p) {
  cudaPointerAttributes at{};
  const bool ok = p && cudaPointerGetAttributes(&at, p) == cudaSuccess && at.type == cudaMemoryTypeHost &&
                  at.devicePointer == p;
  cudaGetLastError();
  return ok;
}

ls_status validate_prefill(const ls_prefill_stream_args* a) {
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->layers >= 1 && a->batch >= 1, "layers and batch must be >= 1");
  LS_REQUIRE(a->max_pages >= 1 && a->max_len >= 1 && a->max_blocks >= 1 && a->num_pages >= 1,
             "max_pages, max_len, max_blocks and num_pages must be >= 1");
  LS_REQUIRE(a->n_slots >= 0 && a->n_slots <= ls::kHbMaxSlots, "n_slots must be in [0, 4096]");
  LS_REQUIRE(a->page_table && a->lens && a->host_keys && a->host_key_scales && a->summaries && a->block_scale,
             "a required pointer is NULL");
  const bool seed = a->n_slots > 0;
  if (seed) {
    LS_REQUIRE(a->host_kv && a->hbuf && a->pos_of_slot && a->slot_of_pos && a->recent_score,
               "hot-buffer seeding needs host_kv, hbuf, pos_of_slot, slot_of_pos and recent_score");
    LS_REQUIRE(a->row_bytes >= 16 && a->row_bytes % 16 == 0, "row_bytes must be a positive multiple of 16");
  }
  for (int l = 0; l < a->layers; ++l) {
    LS_REQUIRE(pinned_host(a->host_keys[l]) && pinned_host(a->host_key_scales[l]),
               "layer %d: host_keys / host_key_scales must be pinned host memory (mapped at the same address)", l);
    LS_REQUIRE(a->summaries[l] && a->block_scale[l], "layer %d: summaries / block_scale is NULL", l);
    if (seed) {
      LS_REQUIRE(pinned_host(a->host_kv[l]) && aligned16(a->host_kv[l]),
                 "layer %d: host_kv must be 16-byte aligned pinned host memory", l);
      LS_REQUIRE(a->hbuf[l] && aligned16(a->hbuf[l]) && a->pos_of_slot[l] && a->slot_of_pos[l] &&
                     a->recent_score[l],
                 "layer %d: a hot-buffer pointer is NULL or misaligned", l);
    }
  }
  return LS_OK;
}

// The copy stream of this host thread on the current device and its events (created once).
struct PrefillStreams {
  cudaStream_t copy = nullptr;
  cudaEvent_t start = nullptr, loaded[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
};
ls_status prefill_streams(PrefillStreams** out) {
  thread_local PrefillStreams per_dev[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return fail(LS_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  PrefillStreams& ps = per_dev[dev];
  if (!ps.copy) {
    bool good = cudaEventCreateWithFlags(&ps.start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2; ++i) {
      good = good && cudaEventCreateWithFlags(&ps.loaded[i], cudaEventDisableTiming) == cudaSuccess;
      good = good && cudaEventCreateWithFlags(&ps.freed[i], cudaEventDisableTiming) == cudaSuccess;
    }
    good = good && cudaStreamCreateWithFlags(&ps.copy, cudaStreamNonBlocking) == cudaSuccess;
    if (!good) {
      ps.copy = nullptr;
      return check_launch("prefill streams");
    }
  }
  *out = &ps;
  return LS_OK;
}

}  // namespace

// An NVTX range around each entry point, so that a profiler's timeline names the calls
// (without a tool attached a push and a pop cost a few nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// =========================================================================================
// C ABI
// =========================================================================================
extern "C" {

const char* ls_version(void) { return LS_VERSION_STRING; }

const char* ls_get_error_string(void) { return g_last_error.c_str(); }

ls_status ls_check_device_status(ls_stream_t stream, uint32_t* flags) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, ls::g_status, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(ls::g_status, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "device status: %s", cudaGetErrorString(e));
  if (flags) *flags = v;
  if (v) return fail(LS_ERR_DEVICE_STATUS, "device status bits 0x%x", v);
  return ok();
}

ls_status ls_set_wait_limit(uint64_t ns) {
  LS_REQUIRE(ns >= 1000 && ns <= 10000000000ull, "the wait limit must be in [1 us, 10 s]");
  const unsigned long long v = ns;
  cudaError_t e = cudaMemcpyToSymbol(ls::g_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "set wait limit: %s", cudaGetErrorString(e));
  return ok();
}

ls_status ls_selftest_bounded_wait(ls_stream_t stream) {
  ls::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
  LS_TRY(check_launch("wait_selftest"));
  return ok();
}

ls_status ls_index_score(const ls_index_score_args* args, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_index_score");
  LS_TRY(validate_index(args, true));
  cudaStream_t st = (cudaStream_t)stream;
  if (args->key_dtype == LS_E4M3 && args->variant == 0) {
    LS_TRY(launch_index_tc(args, 0, nullptr, nullptr, 0, args->scores, args->max_len, nullptr, nullptr, 0, nullptr,
                           0.f, st));
  } else {
    LS_TRY(launch_index_simt(args, st));
  }
  return ok();
}

ls_status ls_topk_select(const ls_topk_args* a, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_topk_select");
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->batch >= 1 && a->k >= 1 && a->k <= 4096, "batch >= 1 and 1 <= k <= 4096 required");
  LS_REQUIRE(a->max_len >= 1 && (a->max_len % 4) == 0, "max_len must be a positive multiple of 4");
  LS_REQUIRE(a->scores && a->lens && a->idx, "scores, lens and idx are required");
  LS_REQUIRE(aligned16(a->scores), "scores must be 16-byte aligned");
  LS_TRY(launch_topk(a->batch, a->k, a->scores, a->max_len, a->lens, 1, 1, a->max_len, nullptr, 0, a->idx,
                     a->sel_score, nullptr, (cudaStream_t)stream, nullptr, 0, a->pos_offset));
  return ok();
}

ls_status ls_build_block_summaries(const ls_index_score_args* keys, uint8_t* summaries, float* block_scale,
                                   int32_t max_blocks, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_build_block_summaries");
  LS_TRY(validate_index(keys, false));
  if (keys->key_dtype != LS_E4M3) return fail(LS_ERR_UNSUPPORTED, "summaries need e4m3 keys");
  LS_REQUIRE(summaries && block_scale && max_blocks >= 1, "summaries, block_scale, max_blocks required");
  ls::SummParams p{};
  p.B = keys->batch; p.max_pages = keys->max_pages; p.max_len = keys->max_len; p.max_blocks = max_blocks;
  p.num_pages = keys->num_pages; p.keys = (const uint8_t*)keys->key_pool; p.ks = keys->key_scale;
  p.page_table = keys->page_table; p.lens = keys->lens; p.summ = summaries; p.bscale = block_scale;
  const int gx = std::min(max_blocks, std::min(keys->max_pages, (keys->max_len + 63) / 64));
  ls::build_summaries_kernel<<<dim3(gx, keys->batch), 128, 0, (cudaStream_t)stream>>>(p);
  LS_TRY(check_launch("build_summaries"));
  return ok();
}

size_t ls_cp_merge_workspace_size(const ls_cp_merge_args* a) {
  if (!a || a->shards < 1 || a->batch < 1 || a->k < 1) return 0;
  const size_t stride = ((size_t)a->shards * a->k + 3) & ~(size_t)3;
  return align256((size_t)a->batch * stride * 4) * 2 + align256((size_t)a->batch * 4);
}

ls_status ls_cp_merge_topk(const ls_cp_merge_args* a, void* workspace, size_t workspace_bytes, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_cp_merge_topk");
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->shards >= 1 && a->batch >= 1 && a->k >= 1 && a->k <= 4096, "shards, batch >= 1, 1 <= k <= 4096");
  LS_REQUIRE((long long)a->shards * a->k <= (1 << 24), "shards * k too large");
  LS_REQUIRE(a->cand_score && a->cand_pos && a->shard_begin && a->shard_end && a->idx,
             "a required pointer is NULL");
  const size_t need = ls_cp_merge_workspace_size(a);
  LS_REQUIRE(workspace && workspace_bytes >= need, "workspace too small (%zu < %zu bytes)", workspace_bytes, need);
  LS_REQUIRE(((uintptr_t)workspace & 255) == 0, "workspace must be 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  const int stride = (a->shards * a->k + 3) & ~3;
  char* w = (char*)workspace;
  float* cscore = (float*)w;
  int* cpos = (int*)(w + align256((size_t)a->batch * stride * 4));
  int* ccount = (int*)(w + 2 * align256((size_t)a->batch * stride * 4));
  ls::CpCompactParams c{};
  c.G = a->shards; c.B = a->batch; c.k = a->k; c.stride = stride; c.cand_score = a->cand_score;
  c.cand_pos = a->cand_pos; c.score = cscore; c.pos = cpos; c.count = ccount;
  ls::cp_compact_kernel<<<a->batch, 256, 0, st>>>(c);
  LS_TRY(check_launch("cp_compact"));
  LS_TRY(launch_topk(a->batch, a->k, cscore, stride, ccount, 1, 1, stride, nullptr, 0, a->idx, a->sel_score,
                     nullptr, st, cpos, stride, nullptr));
  if (a->local_sel) {
    ls::cp_local_sel_kernel<<<dim3((a->k + 255) / 256, a->batch), 256, 0, st>>>(
        a->batch, a->k, a->idx, a->shard_begin, a->shard_end, a->local_sel);
    LS_TRY(check_launch("cp_local_sel"));
  }
  return ok();
}

ls_status ls_attn_merge(const ls_attn_merge_args* a, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_attn_merge");
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->parts >= 1 && a->batch >= 1 && a->heads >= 1 && a->dv >= 4 && a->dv % 4 == 0,
             "parts, batch, heads >= 1 and dv a positive multiple of 4 required");
  LS_REQUIRE(a->o_parts && a->lse_parts && a->o && a->lse, "a required pointer is NULL");
  LS_REQUIRE(a->o_dtype == LS_BF16 || a->o_dtype == LS_F32, "o_dtype must be LS_BF16 or LS_F32");
  LS_REQUIRE(aligned16(a->o_parts) && (a->o_dtype == LS_BF16 ? aligned8(a->o) : aligned16(a->o)),
             "o_parts must be 16-byte aligned, o 8 (bf16) or 16 (f32)");
  ls::MergeParams p{};
  p.G = a->parts; p.B = a->batch; p.H = a->heads; p.DV = a->dv; p.o_f32 = a->o_dtype == LS_F32;
  p.o_parts = a->o_parts; p.lse_parts = a->lse_parts; p.o = a->o; p.lse = a->lse;
  const long long items = (long long)a->batch * a->heads * (a->dv / 4);
  ls::attn_merge_kernel<<<(unsigned)((items + 255) / 256), 256, 0, (cudaStream_t)stream>>>(p);
  LS_TRY(check_launch("attn_merge"));
  return ok();
}

size_t ls_prefill_stream_workspace_size(const ls_prefill_stream_args* args) {
  if (!args) return 0;
  return prefill_layout(args).total;
}

ls_status ls_prefill_stream(const ls_prefill_stream_args* a, void* workspace, size_t workspace_bytes,
                            ls_stream_t stream) {
  NvtxRange nvtx_range("ls_prefill_stream");
  LS_TRY(validate_prefill(a));
  const PrefillLayout l = prefill_layout(a);
  LS_REQUIRE(workspace && workspace_bytes >= l.total, "workspace too small (%zu < %zu bytes)", workspace_bytes,
             l.total);
  LS_REQUIRE(((uintptr_t)workspace & 255) == 0, "workspace must be 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)workspace;
  PrefillStreams* ps = nullptr;
  LS_TRY(prefill_streams(&ps));
  // the staging buffers may still be read by work already queued on `stream`
  cudaEventRecord(ps->start, st);
  cudaStreamWaitEvent(ps->copy, ps->start, 0);
  const size_t key_bytes = (size_t)a->num_pages * 64 * 128, scale_bytes = (size_t)a->num_pages * 64 * 4;
  for (int layer = 0; layer < a->layers; ++layer) {
    const int buf = layer & 1;
    uint8_t* keys = (uint8_t*)(w + l.off_keys[buf]);
    float* scales = (float*)(w + l.off_scales[buf]);
    // copy stream: layer `layer` into buffer `buf`, once the summaries of layer - 2 are done
    if (layer >= 2) cudaStreamWaitEvent(ps->copy, ps->freed[buf], 0);
    cudaError_t e = cudaMemcpyAsync(keys, a->host_keys[layer], key_bytes, cudaMemcpyHostToDevice, ps->copy);
    if (e == cudaSuccess) e = cudaMemcpyAsync(scales, a->host_key_scales[layer], scale_bytes, cudaMemcpyHostToDevice,
                                              ps->copy);
    if (e != cudaSuccess) return fail(LS_ERR_CUDA, "prefill copy (layer %d): %s", layer, cudaGetErrorString(e));
    cudaEventRecord(ps->loaded[buf], ps->copy);
    // `stream`: the layer's summaries from the buffer, then its hot-buffer seed
    cudaStreamWaitEvent(st, ps->loaded[buf], 0);
    ls::SummParams sp{};
    sp.B = a->batch; sp.max_pages = a->max_pages; sp.max_len = a->max_len; sp.max_blocks = a->max_blocks;
    sp.num_pages = a->num_pages; sp.keys = keys; sp.ks = scales; sp.page_table = a->page_table; sp.lens = a->lens;
    sp.summ = a->summaries[layer]; sp.bscale = a->block_scale[layer];
    const int gx = std::min(a->max_blocks, std::min(a->max_pages, (a->max_len + 63) / 64));
    ls::build_summaries_kernel<<<dim3(gx, a->batch), 128, 0, st>>>(sp);
    LS_TRY(check_launch("build_summaries"));
    cudaEventRecord(ps->freed[buf], st);
    if (a->n_slots > 0) {
      int* spos = (int*)(w + l.off_spos);
      int* sslot = (int*)(w + l.off_sslot);
      int* sn = (int*)(w + l.off_sn);
      ls::SeedParams q{};
      q.B = a->batch; q.n_slots = a->n_slots; q.max_len = a->max_len; q.max_pages = a->max_pages; q.lens = a->lens;
      q.pos_of_slot = a->pos_of_slot[layer]; q.slot_of_pos = a->slot_of_pos[layer]; q.recent = a->recent_score[layer];
      q.seed_pos = spos; q.seed_slot = sslot; q.seed_n = sn;
      const int sx = std::max(1, std::min((a->max_len + 255) / 256, (4 * device_sms()) / a->batch));
      ls::seed_hotbuf_kernel<<<dim3(sx, a->batch), 256, 0, st>>>(q);
      LS_TRY(check_launch("seed_hotbuf"));
      ls_gather_args g{};
      g.batch = a->batch; g.k = a->n_slots; g.n_slots = a->n_slots; g.max_pages = a->max_pages;
      g.row_bytes = a->row_bytes; g.num_pages = a->num_pages; g.host_kv = a->host_kv[layer];
      g.page_table = a->page_table; g.miss_pos = spos; g.miss_slot = sslot; g.n_miss = sn; g.hbuf = a->hbuf[layer];
      LS_TRY(launch_gather(&g, st));
    }
  }
  return ok();
}

size_t ls_block_bound_prune_workspace_size(const ls_block_bound_prune_args* args) {
  if (!args) return 0;
  return c2f_layout(args).total;
}

ls_status ls_block_bound_prune(const ls_block_bound_prune_args* args, void* workspace, size_t workspace_bytes,
                               ls_stream_t stream) {
  NvtxRange nvtx_range("ls_block_bound_prune");
  LS_TRY(validate_c2f(args));
  LS_TRY(run_c2f(args, workspace, workspace_bytes, args->survivors, args->n_survivors, nullptr,
                 (cudaStream_t)stream));
  return ok();
}

ls_status ls_hotbuf_resolve(const ls_hotbuf_args* args, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_hotbuf_resolve");
  LS_TRY(validate_hotbuf(args));
  LS_TRY(launch_hotbuf(args, (cudaStream_t)stream));
  return ok();
}

ls_status ls_gather_misses(const ls_gather_args* args, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_gather_misses");
  LS_TRY(validate_gather(args));
  LS_TRY(launch_gather(args, (cudaStream_t)stream));
  return ok();
}

size_t ls_sparse_attn_workspace_size(const ls_sparse_attn_args* args) {
  if (!args) return 0;
  return attn_ws_bytes(args);
}

ls_status ls_sparse_attn_decode(const ls_sparse_attn_args* a, void* workspace, size_t workspace_bytes,
                                ls_stream_t stream) {
  NvtxRange nvtx_range("ls_sparse_attn_decode");
  LS_TRY(validate_attn(a, true));
  LS_TRY(launch_attn(a, a->sel, a->addressing, a->page_table, a->max_pages, a->n_slots, nullptr, a->num_rows,
                     workspace, workspace_bytes, (cudaStream_t)stream, false));
  return ok();
}

size_t ls_decode_step_workspace_size(const ls_decode_step_args* args) {
  if (!args) return 0;
  return step_layout(args).total;
}

ls_status ls_decode_step(const ls_decode_step_args* a, void* workspace, size_t workspace_bytes,
                         ls_stream_t stream) {
  NvtxRange nvtx_range("ls_decode_step");
  LS_REQUIRE(a, "args is NULL");
  LS_REQUIRE(a->k >= 1 && a->k <= 4096, "1 <= k <= 4096 required");
  cudaStream_t st = (cudaStream_t)stream;
  const ls_index_score_args* ix = &a->index;
  LS_TRY(validate_index(ix, false));
  LS_REQUIRE(a->use_c2f || (ix->max_len % 4) == 0, "index.max_len must be a multiple of 4");
  ls_sparse_attn_args at = step_attn_args(a);
  LS_TRY(validate_attn(&at, false));
  if (a->use_hotbuf) {
    LS_REQUIRE(a->pos_of_slot && a->recent_score && a->slot_of_pos && a->host_kv && a->hbuf,
               "hot-buffer state, host_kv and hbuf are required");
    LS_REQUIRE(a->n_slots >= a->k && a->n_slots <= ls::kHbMaxSlots, "need k <= n_slots <= 4096");
    LS_REQUIRE(a->host_num_pages >= 1, "host_num_pages must be >= 1");
    LS_REQUIRE(aligned16(a->host_kv) && aligned16(a->hbuf), "host_kv and hbuf must be 16-byte aligned");
  } else {
    LS_REQUIRE(at.addressing == LS_ROWS_PAGED, "without the hot buffer attention reads the paged pool");
  }
  const StepLayout l = step_layout(a);
  LS_REQUIRE(workspace_bytes >= l.total && (l.total == 0 || workspace), "decode-step workspace too small (%zu < %zu)",
             workspace_bytes, l.total);
  LS_REQUIRE(((uintptr_t)workspace & 255) == 0, "workspace must be 256-byte aligned");
  char* w = (char*)workspace;
  int* idx = a->idx ? a->idx : (int*)(w + l.off_idx);
  float* sel = a->sel_score ? a->sel_score : (float*)(w + l.off_sel);
  ls_event_t* ev = a->events;
  auto rec = [&](int i) {
    if (ev && ev[i]) cudaEventRecord((cudaEvent_t)ev[i], st);
  };
  auto wait_q = [&](cudaStream_t s) {
    if (a->attn_q_ready) cudaStreamWaitEvent(s, (cudaEvent_t)a->attn_q_ready, 0);
  };
  // a1 (+a2) or a3
  int* ready = nullptr;
  int ready_want = 0;
  rec(0);
  if (a->use_c2f) {
    ls_block_bound_prune_args c = step_c2f_args(a, idx, sel);
    LS_TRY(validate_c2f(&c));
    LS_TRY(run_c2f(&c, w + l.off_c2f, l.total - l.off_c2f, a->survivors, a->n_survivors, ev ? ev[1] : nullptr, st));
  } else {
    float* scores = ix->scores ? ix->scores : (float*)(w + l.off_scores);
    // paged path with the tensor-core indexer: per-request completion counts hand each
    // request from the top-k to the attention, and from the attention to the combine; each
    // count is zeroed by the kernel before the one that adds it up
    ready = (!a->use_hotbuf && ix->key_dtype == LS_E4M3 && ix->variant == 0) ? (int*)(w + l.off_ready) : nullptr;
    const bool cand = step_uses_candidates(a);
    ls::IdxTcParams fp{};
    if (cand) {
      fp.filt = (int*)(w + l.off_filt);
      fp.cand_cnt = (int*)(w + l.off_candcnt);
      fp.cand_pos = (int*)(w + l.off_candpos);
      fp.cand_score = (float*)(w + l.off_candscore);
      fp.filt_k = a->k;  // the filter's words: zeroed by the top-k that reads them
    }
    if (ix->key_dtype == LS_E4M3 && ix->variant == 0) {
      LS_TRY(launch_index_tc(ix, 0, nullptr, nullptr, 0, scores, ix->max_len, nullptr, nullptr, 0, nullptr, 0.f, st,
                             -1, 0, ready, cand ? &fp : nullptr));
    } else {
      ls_index_score_args tmp = *ix;
      tmp.scores = scores;
      LS_TRY(launch_index_simt(&tmp, st));
    }
    rec(1);
    int* done = !a->use_hotbuf ? (int*)(w + l.off_done) : nullptr;
    ready_want = ix->max_len <= kTopkRowMaxLen ? 1 : (topk16_supported(st) ? 16 : 8);
    LS_TRY(launch_topk(ix->batch, a->k, scores, ix->max_len, ix->lens, 1, 1, ix->max_len, nullptr, 0, idx, sel,
                       nullptr, st, nullptr, 0, nullptr, done, ready, cand ? &fp : nullptr,
                       cand ? 4 * step_idx_ctas(a) : 0, cand && !a->use_hotbuf ? &a->attn : nullptr));
  }
  void* attn_ws = w + l.off_attn;
  if (a->use_hotbuf) {
    int* sel_slot = a->sel_slot ? a->sel_slot : (int*)(w + l.off_selslot);
    int* mpos = a->miss_pos ? a->miss_pos : (int*)(w + l.off_mpos);
    int* mslot = a->miss_slot ? a->miss_slot : (int*)(w + l.off_mslot);
    int* nmiss = a->n_miss ? a->n_miss : (int*)(w + l.off_nmiss);
    const bool two_pass = overlap_misses(&at);
    const size_t attn_ws_b = attn_ws_bytes(&at, two_pass ? 2 : 1);
    const long long n_rows = (long long)ix->batch * a->n_slots;
    rec(2);
    ls_hotbuf_args h{};
    h.batch = ix->batch; h.k = a->k; h.n_slots = a->n_slots; h.max_len = ix->max_len; h.sel = idx;
    h.sel_score = sel; h.pos_of_slot = a->pos_of_slot; h.recent_score = a->recent_score;
    h.slot_of_pos = a->slot_of_pos; h.sel_slot = sel_slot; h.miss_pos = mpos; h.miss_slot = mslot; h.n_miss = nmiss;
    ls_gather_args g{};
    g.batch = ix->batch; g.k = a->k; g.n_slots = a->n_slots; g.max_pages = ix->max_pages;
    g.row_bytes = at.row_stride * (at.dtype == LS_BF16 ? 2 : 4); g.num_pages = a->host_num_pages;
    g.host_kv = a->host_kv; g.page_table = ix->page_table; g.miss_pos = mpos; g.miss_slot = mslot;
    g.n_miss = nmiss; g.hbuf = a->hbuf;
    if (two_pass) {
      // critical path: classify -> fetch the misses over the host link into staging rows
      // -> attend to them there -> merge.  Beside it: the resident rows' attention, and
      // the victim choice + map update, then the staged rows into their victim slots
      // (victims are never resident selected rows, so nothing here races).
      int* hit_slot = (int*)(w + l.off_hitslot);
      int* cpos = (int*)(w + l.off_cpos);
      int* crow = (int*)(w + l.off_crow);
      int* cn = (int*)(w + l.off_cnmiss);
      int* chit = (int*)(w + l.off_cnhit);
      void* stage = w + l.off_stage;
      LS_TRY(launch_classify(&h, hit_slot, chit, cpos, crow, cn, st));
      rec(3);
      SideStream* ss = nullptr;
      LS_TRY(side_stream(st, &ss));
      cudaEventRecord(ss->fork, st);
      cudaStreamWaitEvent(ss->s[0], ss->fork, 0);
      cudaStreamWaitEvent(ss->s[1], ss->fork, 0);
      LS_TRY(launch_hotbuf(&h, ss->s[0]));
      wait_q(ss->s[1]);
      LS_TRY(launch_attn(&at, hit_slot, LS_ROWS_SLOTS, nullptr, 0, a->n_slots, a->hbuf, n_rows, attn_ws, attn_ws_b,
                         ss->s[1], false, true, 0, 2, false, chit));
      cudaEventRecord(ss->join[1], ss->s[1]);
      ls_gather_args gs = g;
      gs.miss_pos = cpos;
      gs.n_miss = cn;
      LS_TRY(launch_gather(&gs, st, stage));
      rec(4);
      // the staging area as rows: request b's i-th miss at row b*k + i (launched straight
      // after the gather, so that its prologue overlaps the gather's end)
      wait_q(st);
      LS_TRY(launch_attn(&at, crow, LS_ROWS_SLOTS, nullptr, 0, a->k, stage, (long long)ix->batch * a->k, attn_ws,
                         attn_ws_b, st, true, true, 1, 2, false, cn));
      cudaEventRecord(ss->gathered, st);
      cudaStreamWaitEvent(ss->s[0], ss->gathered, 0);
      LS_TRY(launch_copy_staged(&g, stage, ss->s[0]));
      cudaEventRecord(ss->join[0], ss->s[0]);
      cudaStreamWaitEvent(st, ss->join[1], 0);
      LS_TRY(launch_attn_combine(&at, attn_ws, 2, st));
      cudaStreamWaitEvent(st, ss->join[0], 0);
    } else {
      LS_TRY(launch_hotbuf(&h, st));
      rec(3);
      LS_TRY(launch_gather(&g, st));
      rec(4);
      wait_q(st);
      LS_TRY(launch_attn(&at, sel_slot, LS_ROWS_SLOTS, nullptr, 0, a->n_slots, a->hbuf, n_rows, attn_ws, attn_ws_b,
                         st, true));
    }
  } else {
    const size_t attn_ws_b = attn_ws_bytes(&at);
    rec(2);
    rec(3);
    rec(4);
    const int* pt = at.page_table ? at.page_table : ix->page_table;
    const int mp = at.page_table ? at.max_pages : ix->max_pages;
    wait_q(st);
    int* done = !a->use_c2f ? (int*)(w + l.off_done) : nullptr;
    LS_TRY(launch_attn(&at, idx, LS_ROWS_PAGED, pt, mp, 0, nullptr, at.num_rows, attn_ws, attn_ws_b, st, true,
                       true, 0, 1, true, nullptr, done, ready, ready_want));
  }
  rec(5);
  return ok();
}

}  // extern "C"

// =========================================================================================
// Allocation-free attention: the split-KV scratch lives in a fixed device array that the
// library itself provides, for callers that cannot allocate device memory.
// =========================================================================================
namespace {

// Largest split-KV scratch the allocation-free entry point supports.  With 148 SMs the
// split count is floor(148 / (2 * batch)), so the partials of any batch fit in
// 74 * 128 * 512 * 4 B + 74 * 128 * 8 B (about 19 MB).
constexpr size_t kStaticAttnScratchBytes = 20u << 20;

}  // namespace

// One copy per GPU that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_attn_scratch[kStaticAttnScratchBytes];

namespace {

// Id of the calling thread's current CUDA context, unique for the life of the process (a
// context made after another was destroyed -- e.g. after cudaDeviceReset, or one a C
// caller creates itself -- gets a new id, even at the same handle address).  False when no
// context is current or the driver lacks the calls.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();
  });
  CUcontext c = nullptr;
  return get_cur && get_id && get_cur(&c) == CUDA_SUCCESS && c && get_id(c, id) == CUDA_SUCCESS;
}

// Device address of g_attn_scratch in the current context.  In host code the symbol is
// only a host-side stand-in, so the address is asked for once per context (with that
// context current) and cached under the context's id: an address never outlives the
// context it belongs to.  Without a context id the address is looked up on every call.
ls_status static_scratch(void** out) {
  struct Entry {
    unsigned long long ctx;
    void* ptr;
  };
  static Entry cache[64];
  static int n_cached = 0, next_slot = 0;
  static std::mutex mu;
  unsigned long long id = 0;
  if (current_ctx_id(&id)) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_cached; ++i)
      if (cache[i].ctx == id) {
        *out = cache[i].ptr;
        return LS_OK;
      }
  }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
  if (e != cudaSuccess || !p)
    return fail(LS_ERR_CUDA, "cudaGetSymbolAddress(attention scratch): %s", cudaGetErrorString(e));
  // the lookup makes the device's primary context current if none was: ask for the id again
  if (current_ctx_id(&id)) {
    std::lock_guard<std::mutex> lock(mu);
    Entry& slot = n_cached < 64 ? cache[n_cached++] : cache[(next_slot++) & 63];
    slot.ctx = id;
    slot.ptr = p;
  }
  *out = p;
  return LS_OK;
}

}  // namespace

extern "C" ls_status ls_sparse_attn_decode_noalloc(const ls_sparse_attn_args* a, ls_stream_t stream) {
  NvtxRange nvtx_range("ls_sparse_attn_decode_noalloc");
  LS_TRY(validate_attn(a, true));
  const size_t need = attn_ws_bytes(a);
  if (need > kStaticAttnScratchBytes)
    return fail(LS_ERR_INVALID_ARG,
                "allocation-free attention needs %zu bytes of scratch; the built-in scratch holds %zu bytes "
                "(use ls_sparse_attn_decode with a caller workspace)",
                need, kStaticAttnScratchBytes);
  void* ws = nullptr;
  if (need > 0) LS_TRY(static_scratch(&ws));
  LS_TRY(launch_attn(a, a->sel, a->addressing, a->page_table, a->max_pages, a->n_slots, nullptr, a->num_rows, ws,
                     need > 0 ? kStaticAttnScratchBytes : 0, (cudaStream_t)stream, false));
  return ok();
}
