// Host side of the C ABI declared in include/pivot.h: argument checks,
// workspace layout, TMA descriptors and the launch sequence of each call.
//
// Prefill (pivot_index / dense_index), per head pass:
//   proxy_kernel        group means -> fp32 proxies and their three bf16
//                       terms                                 (skipped for dense)
//   proxy_expand_kernel the proxies copied to every position  (per-member scan only)
//   scan_filter_kernel  tcgen05 prefix scan + threshold filter -> spill lists
//   finalize_kernel     exact top-K per row from the spill list
//   fallback_kernel     exact recompute for rows the filter could not settle
// then refine_kernel (Refine only): per-member re-score of the candidate set.
// Decode (pivot_decode_index): proxy_kernel -> decode_scan_kernel ->
// decode_select_kernel -> refine_kernel.
// Consumer (pivot_sparse_attention): sparse_attention_kernel over index rows.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/pivot.h"
#include "attend.cuh"
#include "finalize.cuh"
#include "proxy_decode.cuh"
#include "ptx.cuh"
#include "refine.cuh"
#include "scan.cuh"

namespace {

using namespace pivot;

__device__ int g_status_word;  // per-device kernel status bits

thread_local char g_err[512] = "";

// Limit of the kernels' bounded waits (pivot_set_wait_limit); 0 = the default.
std::atomic<unsigned long long> g_wait_ns{0};
unsigned long long wait_limit_ns() {
  const unsigned long long v = g_wait_ns.load();
  return v ? v : kWaitNs;
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

// ---------------------------------------------------------------- launch trace
// Optional: every kernel launch of the calling thread is bracketed by two CUDA
// events on its stream; pivot_trace_collect() turns them into per-kernel times.
struct TraceRec {
  const char* name;
  cudaEvent_t a, b;
};
thread_local bool g_trace_on = false;
thread_local std::vector<TraceRec> g_trace;
thread_local std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct TraceScope {
  TraceRec rec{nullptr, nullptr, nullptr};
  cudaStream_t st;
  TraceScope(const char* name, cudaStream_t s) : st(s) {
    if (!g_trace_on) return;
    rec.name = name;
    rec.a = pool_event();
    rec.b = pool_event();
    cudaEventRecord(rec.a, st);
  }
  ~TraceScope() {
    if (!rec.name) return;
    cudaEventRecord(rec.b, st);
    g_trace.push_back(rec);
  }
};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sms = 0;
  int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(PIVOT_ERR_UNSUPPORTED, "no CUDA device available");
  if (dev < 0 || dev >= kMaxDevices) return fail(PIVOT_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
    if (d.supported) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess)
        return fail(PIVOT_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(cudaGetLastError()));
      d.status = static_cast<int*>(p);
    }
    d.ready = true;
  }
  if (!d.supported) return fail(PIVOT_ERR_UNSUPPORTED, "this library needs an sm_100 (B200) device");
  *out = &d;
  return PIVOT_OK;
}

// ---------------------------------------------------------------- TMA descriptors
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

// View of a [rows][H][d] bf16 tensor starting at `base` (which may point at a
// later head), covering `heads` heads; box = 64 channels x 1 head x box_rows
// rows, 128-byte swizzle.
int make_rows_map(CUtensorMap* m, const void* base, int rows, int heads, int H, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PIVOT_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PIVOT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PIVOT_OK;
}

// ---------------------------------------------------------------- workspace layout
constexpr size_t kAlign = 256;
constexpr size_t kSpillBudget = size_t(8) << 30;  // spill bytes per head pass

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
  // sizes: G = scan rows per head (groups; positions for dense and the
  // per-member scan), Gg = groups (proxy rows)
  int G, Gg, cap, S, K_sel, heads_per_pass, nfb;
  // offsets
  size_t off_proxy, off_proxy_e, off_spill, off_cnt, off_fb, off_fblist, off_fbscratch, off_cand, off_miss, total;
};

// Sample stride and spill capacity for a select of K_sel keys per row over
// prefixes up to L keys.
void filter_shape(int K_sel, int L, int* cap, int* S) {
  const int BN = 128;  // keys per scan tile
  int c = std::max(2 * K_sel, 4 * BN);
  int s = std::max(1, std::min(16, c / BN));
  // at most 511 sampled tiles per row, so a row's sample fits 16-bit bin counts
  const int min_s = (L + BN * 511 - 1) / (BN * 511);
  s = std::max(s, min_s);
  c = std::max(c, s * BN);
  *cap = (c + 7) / 8 * 8;
  *S = s;
}

// Refine's miss list: a counter, then one (item, member) entry per member of
// every unit (the most the select can hand to the fallback).
size_t miss_cap(size_t units, int g) { return units * static_cast<size_t>((g + 15) / 16) * 16; }
size_t miss_bytes(size_t units, int g) { return up(sizeof(int)) + up(miss_cap(units, g) * sizeof(int2)); }

// The mode argument: PIVOT_REFINE or PIVOT_REUSE, optionally OR-ed with
// PIVOT_PROXY_BF16 and (Refine) PIVOT_PER_MEMBER_SCAN.
int base_mode(int mode) { return mode & ~static_cast<int>(PIVOT_PROXY_BF16 | PIVOT_PER_MEMBER_SCAN); }
bool proxy_bf16(int mode) { return (mode & PIVOT_PROXY_BF16) != 0; }
bool per_member_scan(int mode) { return (mode & PIVOT_PER_MEMBER_SCAN) != 0; }

Plan plan_prefill(int L, int H, int d, int g, int top_k, int Kc, int mode_bits, bool dense, int sms) {
  const int mode = base_mode(mode_bits);
  const bool pm = !dense && mode == PIVOT_REFINE && per_member_scan(mode_bits);
  Plan p{};
  p.Gg = dense ? L : (L + g - 1) / g;
  p.G = pm ? L : p.Gg;
  p.K_sel = (dense || mode == PIVOT_REUSE) ? top_k : Kc;
  filter_shape(p.K_sel, L, &p.cap, &p.S);
  const size_t per_head_spill = static_cast<size_t>(p.G) * p.cap * sizeof(uint2);
  p.heads_per_pass = static_cast<int>(std::max<size_t>(1, std::min<size_t>(H, kSpillBudget / per_head_spill)));
  p.nfb = 2 * std::max(1, sms);
  const size_t rows_pass = static_cast<size_t>(p.heads_per_pass) * p.G;
  size_t o = 0;
  // fp32 proxies [Gg][H][d], then their bf16 terms [3][Gg][H][d]; for the
  // per-member scan the same per position, [L][H][d] and [3][L][H][d]
  p.off_proxy = o;
  o += dense ? 0 : up(static_cast<size_t>(p.Gg) * H * d * 4) + up(static_cast<size_t>(3) * p.Gg * H * d * 2);
  p.off_proxy_e = o;
  o += pm ? up(static_cast<size_t>(L) * H * d * 4) + up(static_cast<size_t>(3) * L * H * d * 2) : 0;
  p.off_spill = o;
  o += up(rows_pass * p.cap * sizeof(uint2));
  p.off_cnt = o;
  o += up(rows_pass * sizeof(int4));
  p.off_fb = o;
  o += up(sizeof(int));
  p.off_fblist = o;
  o += up(rows_pass * sizeof(int));
  p.off_fbscratch = o;
  o += up(static_cast<size_t>(p.nfb) * L * sizeof(uint32_t));
  p.off_cand = o;
  o += (!dense && mode == PIVOT_REFINE) ? up(static_cast<size_t>(H) * p.G * cand_row_words(Kc) * sizeof(int32_t)) : 0;
  p.off_miss = o;
  o += (!dense && mode == PIVOT_REFINE) ? miss_bytes(static_cast<size_t>(H) * p.G, pm ? 1 : g) : 0;
  p.total = o;
  return p;
}

uint32_t tmem_cols_for(int Kc) {
  const int need = 16 * ((Kc + 127) / 128);
  uint32_t c = 32;
  while (static_cast<int>(c) < need) c <<= 1;
  return c;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


int check_common(const void* q, const void* k, int H, int d, int top_k, int Kc, int mode, const void* out) {
  if (!q || !k || !out) return fail(PIVOT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(out))
    return fail(PIVOT_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (H < 1) return fail(PIVOT_ERR_INVALID_ARG, "H must be >= 1");
  if (d != 64 && d != 128) return fail(PIVOT_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", d);
  if (top_k < 1 || Kc < top_k || Kc > 4096)
    return fail(PIVOT_ERR_INVALID_ARG, "need 1 <= top_k <= Kc <= 4096 (top_k=%d, Kc=%d)", top_k, Kc);
  if (base_mode(mode) != PIVOT_REFINE && base_mode(mode) != PIVOT_REUSE)
    return fail(PIVOT_ERR_INVALID_ARG,
                "mode must be PIVOT_REFINE or PIVOT_REUSE, optionally | PIVOT_PROXY_BF16 (| PIVOT_PER_MEMBER_SCAN)");
  if (per_member_scan(mode) && base_mode(mode) != PIVOT_REFINE)
    return fail(PIVOT_ERR_INVALID_ARG, "PIVOT_PER_MEMBER_SCAN applies to PIVOT_REFINE only");
  return PIVOT_OK;
}

#define CUDA_TRY(expr)                                                                       \
  do {                                                                                       \
    cudaError_t e_ = (expr);                                                                 \
    if (e_ != cudaSuccess) return fail(PIVOT_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

template <int D>
int launch_scan(const CUtensorMap& tmP, const CUtensorMap& tmK, const ScanParams& sp, int heads, cudaStream_t st) {
  using C = ScanCfg<D>;
  CUDA_TRY(cudaFuncSetAttribute(scan_filter_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
  TraceScope tr("scan_filter", st);
  scan_filter_kernel<D><<<heads * sp.tiles_per_head, C::THREADS, C::SMEM, st>>>(tmP, tmK, sp);
  CUDA_TRY(cudaGetLastError());
  return PIVOT_OK;
}

// Refine, then the exact redo of the members its select could not settle.
// `miss` points at the workspace region sized by miss_bytes(units, g).
template <int D>
int launch_refine(RefineParams rp, int units, int sms, uint8_t* miss, cudaStream_t st) {
  const int smem = RefineCfg<D>::smem_bytes(rp.Kc);
  // a paged decode cache looks each candidate's key row up in the block table
  const bool paged = rp.ci.block_table != nullptr;
  auto kern = paged ? refine_kernel<D, true> : refine_kernel<D, false>;
  CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  rp.nbatch = (rp.g + 15) / 16;
  rp.n_items = units * rp.nbatch;
  rp.miss_count = reinterpret_cast<int*>(miss);
  rp.miss_list = reinterpret_cast<int2*>(miss + up(sizeof(int)));
  rp.miss_cap = static_cast<int>(std::min<size_t>(miss_cap(units, rp.g), 0x7FFFFFFF));
  CUDA_TRY(cudaMemsetAsync(rp.miss_count, 0, sizeof(int), st));
  // persistent: one CTA per SM walks the items
  const int grid = std::max(1, std::min(rp.n_items, sms));
  {
    TraceScope tr("refine", st);
    kern<<<grid, RefineCfg<D>::NT, smem, st>>>(rp);
  }
  CUDA_TRY(cudaGetLastError());
  const int fsmem = (2 * cand_row_words(rp.Kc) + 2 * rp.top_k) * 4;
  CUDA_TRY(cudaFuncSetAttribute(refine_fallback_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, fsmem));
  {
    TraceScope tr("refine_fallback", st);
    refine_fallback_kernel<D><<<2 * std::max(1, sms), kRfbNT, fsmem, st>>>(rp);
  }
  CUDA_TRY(cudaGetLastError());
  return PIVOT_OK;
}

// Shared prefill driver (PIVOT Refine/Reuse, and dense when `dense`).
// Copies candidate rows ([H][G][CW]) to the layout out[unit][h][Kc]:
// ascending key indices, -1 padding.  Row
// (h, u) holds n = min(Kc, bound) candidates; bound is the Refine scan bound
// (prefill: the group's last position; decode: n_b + g - 1, or no candidates
// for a sequence the decode scan skipped).
__global__ void cand_export_kernel(const int32_t* __restrict__ cand, int32_t* __restrict__ out, int G, int H,
                                   int Kc, int g, int L, CacheIndex ci, int max_seqlen) {
  const int h = blockIdx.x / G, u = blockIdx.x % G;
  int bound;
  if (!ci.decode()) {
    bound = min(u * g + g, L) - 1;
  } else {
    const int len = ci.len(u);
    bound = (len > max_seqlen || len < g) ? 0 : len - 1;
  }
  const int n = min(Kc, max(bound, 0));
  const int32_t* row = cand + (static_cast<long long>(h) * G + u) * cand_row_words(Kc);
  int32_t* dst = out + (static_cast<long long>(u) * H + h) * Kc;
  for (int t = threadIdx.x; t < Kc; t += blockDim.x) dst[t] = t < n ? row[t] : -1;
}

int run_prefill(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode_bits,
                bool dense, int32_t* out, float* out_scores, float* out_proxy, int32_t* out_cand, void* ws,
                size_t ws_bytes, cudaStream_t st) {
  const int mode = base_mode(mode_bits);
  if (L < 1) return fail(PIVOT_ERR_INVALID_ARG, "L must be >= 1");
  if (!dense && g < 1) return fail(PIVOT_ERR_INVALID_ARG, "g must be >= 1");
  if (static_cast<long long>(L) * H * d >= (1ll << 40)) return fail(PIVOT_ERR_INVALID_ARG, "tensor too large");
  if (L >= (1 << 30)) return fail(PIVOT_ERR_INVALID_ARG, "L too large");
  if (out_scores && !aligned16(out_scores)) return fail(PIVOT_ERR_INVALID_ARG, "out_scores must be 16-byte aligned");
  if (out_proxy && !aligned16(out_proxy)) return fail(PIVOT_ERR_INVALID_ARG, "out_proxy must be 16-byte aligned");
  if (out_cand && mode != PIVOT_REFINE)
    return fail(PIVOT_ERR_INVALID_ARG, "out_cand is only produced in PIVOT_REFINE mode");
  if (per_member_scan(mode_bits) && (dense || mode != PIVOT_REFINE))
    return fail(PIVOT_ERR_INVALID_ARG, "PIVOT_PER_MEMBER_SCAN applies to PIVOT_REFINE only");
  const bool pm = per_member_scan(mode_bits);
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const Plan pl = plan_prefill(L, H, d, dense ? 1 : g, top_k, Kc, mode_bits, dense, dev->sms);
  if (!ws || ws_bytes < pl.total)
    return fail(PIVOT_ERR_WORKSPACE, "workspace too small: need %zu bytes, got %zu", pl.total, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return fail(PIVOT_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  uint8_t* w = static_cast<uint8_t*>(ws);
  // scan operand: the queries themselves (dense), else the proxies' bf16
  // terms (per group; for the per-member scan copied to every position)
  float* P32g = dense ? nullptr : reinterpret_cast<float*>(w + pl.off_proxy);
  uint16_t* P3g = dense ? nullptr : reinterpret_cast<uint16_t*>(w + pl.off_proxy + up(static_cast<size_t>(pl.Gg) * H * d * 4));
  float* P32e = pm ? reinterpret_cast<float*>(w + pl.off_proxy_e) : nullptr;
  uint16_t* P3e = pm ? reinterpret_cast<uint16_t*>(w + pl.off_proxy_e + up(static_cast<size_t>(L) * H * d * 4)) : nullptr;
  const float* P32 = pm ? P32e : P32g;
  const uint16_t* P = dense ? static_cast<const uint16_t*>(q) : (pm ? P3e : P3g);
  const int gg = dense ? 1 : g;
  const int g_scan = pm ? 1 : gg;   // members per scan row
  const bool refine = !dense && mode == PIVOT_REFINE;
  // a proxy of one member is that member's bf16 query: its mid and lo terms are zero
  const int nterms = (dense || gg == 1 || proxy_bf16(mode_bits)) ? 1 : 3;

  if (!dense) {
    const long long n = static_cast<long long>(pl.Gg) * H * (d / 8);
    TraceScope tr("proxy", st);
    proxy_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        static_cast<const uint16_t*>(q), P32g, P3g, pl.Gg, H, d, gg, L, 0, proxy_bf16(mode_bits) ? 1 : 0);
    CUDA_TRY(cudaGetLastError());
    if (out_proxy)
      CUDA_TRY(cudaMemcpyAsync(out_proxy, P32g, static_cast<size_t>(pl.Gg) * H * d * 4, cudaMemcpyDeviceToDevice, st));
  }
  if (pm) {
    const long long n = static_cast<long long>(L) * H * (d / 8);
    TraceScope tr("proxy_expand", st);
    proxy_expand_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(P32g, P3g, P32e, P3e, pl.Gg, L, H,
                                                                                   d, g);
    CUDA_TRY(cudaGetLastError());
  }

  for (int h0 = 0; h0 < H; h0 += pl.heads_per_pass) {
    const int nh = std::min(pl.heads_per_pass, H - h0);
    // TMA views start at head h0 so that the kernels' head index is pass-local.
    const uint16_t* Ph = P + static_cast<size_t>(h0) * d;
    const uint16_t* Kh = static_cast<const uint16_t*>(k) + static_cast<size_t>(h0) * d;
    CUtensorMap tmP, tmK;
    // the proxy view spans the three term tensors: term t's rows start at t*G
    if (int rc = make_rows_map(&tmP, Ph, dense ? pl.G : 3 * pl.G, nh, H, d, 128)) return rc;
    if (int rc = make_rows_map(&tmK, Kh, L, nh, H, d, ScanCfg<128>::BN)) return rc;
    ScanParams sp{};
    sp.G = pl.G;
    sp.L = L;
    sp.H = H;
    sp.g = g_scan;
    // Refine: row i sees j < last(i); Reuse and dense: j < i*g; the
    // per-member scan: position i sees j < i
    sp.bound_kind = (refine && !pm) ? 0 : 1;
    sp.K_sel = pl.K_sel;
    sp.cap = pl.cap;
    sp.S = pl.S;
    sp.tiles_per_head = (pl.G + ScanCfg<128>::BM - 1) / ScanCfg<128>::BM;
    sp.nterms = nterms;
    sp.spill = reinterpret_cast<uint2*>(w + pl.off_spill);
    sp.cnt = reinterpret_cast<int4*>(w + pl.off_cnt);
    sp.status = dev->status;
    sp.wait_ns = wait_limit_ns();
    int rc = (d == 128) ? launch_scan<128>(tmP, tmK, sp, nh, st) : launch_scan<64>(tmP, tmK, sp, nh, st);
    if (rc) return rc;

    FinalizeParams fp{};
    fp.G = pl.G;
    fp.L = L;
    fp.H = H;
    fp.g = g_scan;
    fp.bound_kind = sp.bound_kind;
    fp.K_sel = pl.K_sel;
    fp.cap = pl.cap;
    fp.width = refine ? cand_row_words(Kc) : top_k;
    fp.broadcast = refine ? 0 : 1;
    fp.spill = sp.spill;
    fp.cnt = sp.cnt;
    // Head-local row ids: shift the output bases by h0 heads.
    fp.cand = refine ? reinterpret_cast<int32_t*>(w + pl.off_cand) + static_cast<size_t>(h0) * pl.G * cand_row_words(Kc)
                     : nullptr;
    fp.out = refine ? nullptr : out + static_cast<size_t>(h0) * top_k;
    fp.out_scores = (refine || !out_scores) ? nullptr : out_scores + static_cast<size_t>(h0) * top_k;
    fp.fb_list = reinterpret_cast<int*>(w + pl.off_fblist);
    fp.fb_count = reinterpret_cast<int*>(w + pl.off_fb);
    fp.status = dev->status;
    fp.proxy32 = dense ? nullptr : P32 + static_cast<size_t>(h0) * d;
    fp.proxy16 = dense ? Ph : nullptr;
    fp.keys = Kh;
    fp.d = d;
    fp.fb_scratch = reinterpret_cast<uint32_t*>(w + pl.off_fbscratch);
    CUDA_TRY(cudaMemsetAsync(fp.fb_count, 0, sizeof(int), st));
    // candidate rows are written straight from the select; index rows are staged
    const int fin_smem = pl.cap * 8 + (refine ? 0 : pl.K_sel * 8);
    CUDA_TRY(cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fin_smem));
    {
      TraceScope tr("finalize", st);
      finalize_kernel<<<static_cast<unsigned>(nh * pl.G), kFinNT, fin_smem, st>>>(fp);
    }
    CUDA_TRY(cudaGetLastError());
    const int fb_smem = pl.K_sel * 8;
    CUDA_TRY(cudaFuncSetAttribute(fallback_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fb_smem));
    {
      TraceScope tr("fallback", st);
      fallback_kernel<<<pl.nfb, kFbNT, fb_smem, st>>>(fp);
    }
    CUDA_TRY(cudaGetLastError());
  }

  if (refine) {
    RefineParams rp{};
    rp.q = static_cast<const uint16_t*>(q);
    rp.keys = static_cast<const uint16_t*>(k);
    rp.cand = reinterpret_cast<const int32_t*>(w + pl.off_cand);
    rp.out = out;
    rp.out_scores = out_scores;
    rp.ci = CacheIndex{};
    rp.G = pl.G;
    rp.L = L;
    rp.H = H;
    rp.g = g_scan;   // the per-member scan: one member per unit, its own candidate row
    rp.top_k = top_k;
    rp.Kc = Kc;
    rp.d = d;
    rp.tmem_cols = tmem_cols_for(Kc);
    rp.status = dev->status;
    rp.wait_ns = wait_limit_ns();
    if (out_cand) {
      cand_export_kernel<<<static_cast<unsigned>(H * pl.G), 256, 0, st>>>(rp.cand, out_cand, pl.G, H, Kc, g_scan,
                                                                          L, CacheIndex{}, 0);
      CUDA_TRY(cudaGetLastError());
    }
    uint8_t* miss = w + pl.off_miss;
    int rc = (d == 128) ? launch_refine<128>(rp, H * pl.G, dev->sms, miss, st)
                        : launch_refine<64>(rp, H * pl.G, dev->sms, miss, st);
    if (rc) return rc;
  }
  return PIVOT_OK;
}

size_t decode_ws_size(int B, int H, int d, int g, int Kc, int mode, int max_seqlen) {
  mode = base_mode(mode);
  size_t o = up(static_cast<size_t>(B) * H * d * 4);                        // fp32 proxies
  o += up(static_cast<size_t>(H) * B * max_seqlen * sizeof(uint32_t));       // order keys
  if (mode == PIVOT_REFINE) o += up(static_cast<size_t>(H) * B * cand_row_words(Kc) * sizeof(int32_t));
  if (mode == PIVOT_REFINE) o += miss_bytes(static_cast<size_t>(H) * B, g);
  return o;
}

// The packed decode cache of the cu_seqlens entry points.
CacheIndex packed(const int32_t* cu) { return CacheIndex{cu, nullptr, nullptr, 0, 0}; }

int check_decode(const void* q, const void* kc, const CacheIndex& ci, int B, int H, int d, int g, int top_k, int Kc,
                 int mode, int max_seqlen, const void* out, const void* out_scores) {
  if (int rc = check_common(q, kc, H, d, top_k, Kc, mode, out)) return rc;
  if (!ci.cu && !(ci.seqlens && ci.block_table))
    return fail(PIVOT_ERR_INVALID_ARG, "null cu_seqlens (packed cache) or seqlens / block_table (paged cache)");
  if (!ci.cu) {
    if (ci.max_pages < 1 || ci.log2_page < 0 || ci.log2_page > 20)
      return fail(PIVOT_ERR_INVALID_ARG, "need max_pages >= 1 and a page size that is a power of two <= 2^20");
    if ((static_cast<long long>(ci.max_pages) << ci.log2_page) < max_seqlen)
      return fail(PIVOT_ERR_INVALID_ARG, "max_seqlen exceeds max_pages * page_size");
  }
  if (per_member_scan(mode)) return fail(PIVOT_ERR_INVALID_ARG, "PIVOT_PER_MEMBER_SCAN applies to the prefill entry points only");
  if (B < 1 || g < 1 || max_seqlen < g) return fail(PIVOT_ERR_INVALID_ARG, "need B >= 1, g >= 1, max_seqlen >= g");
  if (max_seqlen >= (1 << 30)) return fail(PIVOT_ERR_INVALID_ARG, "max_seqlen too large");
  if (out_scores && !aligned16(out_scores)) return fail(PIVOT_ERR_INVALID_ARG, "out_scores must be 16-byte aligned");
  return PIVOT_OK;
}

int run_decode(const void* q, const void* kc, const CacheIndex& ci, int B, int H, int d, int g, int top_k, int Kc,
               int mode_bits, int max_seqlen, int32_t* out, float* out_scores, float* out_proxy, int32_t* out_cand,
               void* ws, size_t ws_bytes, cudaStream_t st) {
  if (int rc = check_decode(q, kc, ci, B, H, d, g, top_k, Kc, mode_bits, max_seqlen, out, out_scores)) return rc;
  const int mode = base_mode(mode_bits);
  if (out_proxy && !aligned16(out_proxy)) return fail(PIVOT_ERR_INVALID_ARG, "out_proxy must be 16-byte aligned");
  if (out_cand && mode != PIVOT_REFINE)
    return fail(PIVOT_ERR_INVALID_ARG, "out_cand is only produced in PIVOT_REFINE mode");
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const size_t need = decode_ws_size(B, H, d, g, Kc, mode, max_seqlen);
  if (!ws || ws_bytes < need) return fail(PIVOT_ERR_WORKSPACE, "workspace too small: need %zu bytes", need);
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return fail(PIVOT_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* P = reinterpret_cast<float*>(w);
  uint32_t* scores = reinterpret_cast<uint32_t*>(w + up(static_cast<size_t>(B) * H * d * 4));
  int32_t* cand = reinterpret_cast<int32_t*>(w + up(static_cast<size_t>(B) * H * d * 4) +
                                             up(static_cast<size_t>(H) * B * max_seqlen * sizeof(uint32_t)));
  const long long n = static_cast<long long>(B) * H * (d / 8);
  {
    // the decode scan multiplies by the fp32 proxy directly: no bf16 terms
    TraceScope tr("proxy", st);
    proxy_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(static_cast<const uint16_t*>(q), P, nullptr,
                                                                          B, H, d, g, 0, 1,
                                                                          proxy_bf16(mode_bits) ? 1 : 0);
  }
  CUDA_TRY(cudaGetLastError());
  if (out_proxy) CUDA_TRY(cudaMemcpyAsync(out_proxy, P, static_cast<size_t>(B) * H * d * 4, cudaMemcpyDeviceToDevice, st));
  DecodeParams dp{};
  dp.kcache = static_cast<const uint16_t*>(kc);
  dp.P = P;
  dp.ci = ci;
  dp.scores = scores;
  dp.cand = mode == PIVOT_REFINE ? cand : nullptr;
  dp.out = out;
  dp.out_scores = mode == PIVOT_REUSE ? out_scores : nullptr;
  dp.B = B;
  dp.H = H;
  dp.d = d;
  dp.g = g;
  dp.mode = mode;
  dp.K_sel = mode == PIVOT_REFINE ? Kc : top_k;
  dp.width = mode == PIVOT_REFINE ? Kc : top_k;
  dp.max_seqlen = max_seqlen;
  dp.status = dev->status;
  dim3 grid((max_seqlen + kDecChunk - 1) / kDecChunk, H, B);
  {
  TraceScope tr("decode_scan", st);
  const bool paged = ci.cu == nullptr;
  if (d == 128)
    (paged ? decode_scan_kernel<128, true> : decode_scan_kernel<128, false>)<<<grid, kDecNT, 0, st>>>(dp);
  else
    (paged ? decode_scan_kernel<64, true> : decode_scan_kernel<64, false>)<<<grid, kDecNT, 0, st>>>(dp);
  }
  CUDA_TRY(cudaGetLastError());
  const int sel_smem = dp.K_sel * 8;
  CUDA_TRY(cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sel_smem));
  {
    TraceScope tr("decode_select", st);
    decode_select_kernel<<<B * H, kDecSelNT, sel_smem, st>>>(dp);
  }
  CUDA_TRY(cudaGetLastError());
  if (mode == PIVOT_REFINE) {
    RefineParams rp{};
    rp.q = static_cast<const uint16_t*>(q);
    rp.keys = static_cast<const uint16_t*>(kc);
    rp.cand = cand;
    rp.out = out;
    rp.out_scores = out_scores;
    rp.ci = ci;
    rp.max_seqlen = max_seqlen;
    rp.G = B;
    rp.L = 0;
    rp.H = H;
    rp.g = g;
    rp.top_k = top_k;
    rp.Kc = Kc;
    rp.d = d;
    rp.tmem_cols = tmem_cols_for(Kc);
    rp.status = dev->status;
    rp.wait_ns = wait_limit_ns();
    if (out_cand) {
      cand_export_kernel<<<static_cast<unsigned>(H * B), 256, 0, st>>>(cand, out_cand, B, H, Kc, g, 0, ci, max_seqlen);
      CUDA_TRY(cudaGetLastError());
    }
    uint8_t* miss = reinterpret_cast<uint8_t*>(cand) + up(static_cast<size_t>(H) * B * cand_row_words(Kc) * sizeof(int32_t));
    int rc = (d == 128) ? launch_refine<128>(rp, H * B, dev->sms, miss, st)
                        : launch_refine<64>(rp, H * B, dev->sms, miss, st);
    if (rc) return rc;
  }
  return PIVOT_OK;
}

// Runs `body(ws, bytes)` with a stream-ordered temporary allocation.
template <class F>
int with_temp_workspace(size_t bytes, cudaStream_t st, F body) {
  void* ws = nullptr;
  CUDA_TRY(cudaMallocAsync(&ws, std::max<size_t>(bytes, kAlign), st));
  const int rc = body(ws, bytes);
  const cudaError_t e = cudaFreeAsync(ws, st);
  if (rc) return rc;
  if (e != cudaSuccess) return fail(PIVOT_ERR_CUDA, "cudaFreeAsync: %s", cudaGetErrorString(e));
  return PIVOT_OK;
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

// ---------------------------------------------------------------- no-allocation decode
// Scratch for pivot_decode_index_noalloc: a fixed device array that every GPU
// loading this library holds until the process exits.  Host code must not pass
// the symbol itself to a kernel (on the host it is only a stand-in); its device
// address is looked up once per device below.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
void* g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call per device, with that device current).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(PIVOT_ERR_UNSUPPORTED, "no usable CUDA device");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(PIVOT_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return PIVOT_OK;
}
}  // namespace

extern "C" {

int pivot_decode_index_noalloc(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d,
                               int g, int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx,
                               float* out_scores, void* stream) {
  if (int rc = check_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, out_scores))
    return rc;
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const size_t need = decode_ws_size(B, H, d, g, Kc, mode, max_seqlen);
  if (need > kNoAllocScratchBytes)
    return fail(PIVOT_ERR_WORKSPACE,
                "pivot_decode_index_noalloc: this call needs %zu bytes of scratch, more than the %zu-byte static "
                "maximum (use pivot_decode_index_ws with a caller workspace)",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  // Nothing in the decode scratch has to start at zero: every word is written
  // before it is read within the call.
  return run_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, out_scores, nullptr,
                    nullptr, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}


size_t pivot_workspace_size(int L, int H, int d, int g, int top_k, int Kc, int mode) {
  if (L < 1 || H < 1 || g < 1 || top_k < 1 || Kc < top_k) return 0;
  return plan_prefill(L, H, d, g, top_k, Kc, mode, false, device_sms()).total;
}

size_t dense_workspace_size(int L, int H, int d, int top_k) {
  if (L < 1 || H < 1 || top_k < 1) return 0;
  return plan_prefill(L, H, d, 1, top_k, top_k, PIVOT_REUSE, true, device_sms()).total;
}

size_t pivot_decode_workspace_size(int B, int H, int d, int g, int top_k, int Kc, int mode, int max_seqlen) {
  (void)top_k;
  if (B < 1 || H < 1 || max_seqlen < 1) return 0;
  return decode_ws_size(B, H, d, g, Kc, mode, max_seqlen);
}

int pivot_index_ws(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                   int32_t* out_idx, float* out_scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (int rc = check_common(q, k, H, d, top_k, Kc, mode, out_idx)) return rc;
  return run_prefill(q, k, L, H, d, g, top_k, Kc, mode, false, out_idx, out_scores, nullptr, nullptr, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pivot_index_ex(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                   int32_t* out_idx, float* out_scores, float* out_proxy, int32_t* out_cand, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (int rc = check_common(q, k, H, d, top_k, Kc, mode, out_idx)) return rc;
  return run_prefill(q, k, L, H, d, g, top_k, Kc, mode, false, out_idx, out_scores, out_proxy, out_cand, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pivot_index(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                int32_t* out_idx, void* stream) {
  if (int rc = check_common(q, k, H, d, top_k, Kc, mode, out_idx)) return rc;
  if (L < 1 || g < 1) return fail(PIVOT_ERR_INVALID_ARG, "need L >= 1 and g >= 1");
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = plan_prefill(L, H, d, g, top_k, Kc, mode, false, dev->sms).total;
  return with_temp_workspace(bytes, st, [&](void* ws, size_t n) {
    return run_prefill(q, k, L, H, d, g, top_k, Kc, mode, false, out_idx, nullptr, nullptr, nullptr, ws, n, st);
  });
}

int dense_index_ws(const void* q, const void* k, int L, int H, int d, int top_k, int32_t* out_idx,
                   float* out_scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (int rc = check_common(q, k, H, d, top_k, top_k, PIVOT_REUSE, out_idx)) return rc;
  return run_prefill(q, k, L, H, d, 1, top_k, top_k, PIVOT_REUSE, true, out_idx, out_scores, nullptr, nullptr,
                     workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int dense_index(const void* q, const void* k, int L, int H, int d, int top_k, int32_t* out_idx, void* stream) {
  if (int rc = check_common(q, k, H, d, top_k, top_k, PIVOT_REUSE, out_idx)) return rc;
  if (L < 1) return fail(PIVOT_ERR_INVALID_ARG, "L must be >= 1");
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = plan_prefill(L, H, d, 1, top_k, top_k, PIVOT_REUSE, true, dev->sms).total;
  return with_temp_workspace(bytes, st, [&](void* ws, size_t n) {
    return run_prefill(q, k, L, H, d, 1, top_k, top_k, PIVOT_REUSE, true, out_idx, nullptr, nullptr, nullptr, ws,
                       n, st);
  });
}

int pivot_decode_index_ws(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d,
                          int g, int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx,
                          float* out_scores, void* workspace, size_t workspace_bytes, void* stream) {
  return run_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, out_scores, nullptr,
                    nullptr, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pivot_sparse_attention(const void* q, const void* k, const void* v, const int32_t* idx,
                           const int32_t* cu_seqlens, int R, int H, int d, int g, int top_k, float* out,
                           void* stream) {
  if (!q || !k || !v || !idx || !out) return fail(PIVOT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out))
    return fail(PIVOT_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (R < 1 || H < 1 || top_k < 1 || (cu_seqlens && g < 1))
    return fail(PIVOT_ERR_INVALID_ARG, "need R >= 1, H >= 1, top_k >= 1 (and g >= 1 with cu_seqlens)");
  if (static_cast<long long>(R) * H >= (1ll << 31)) return fail(PIVOT_ERR_INVALID_ARG, "R * H too large");
  if (d != 64 && d != 128) return fail(PIVOT_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", d);
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  AttendParams ap{};
  ap.q = static_cast<const uint16_t*>(q);
  ap.k = static_cast<const uint16_t*>(k);
  ap.v = static_cast<const uint16_t*>(v);
  ap.idx = idx;
  ap.cu = cu_seqlens;
  ap.out = out;
  ap.R = R;
  ap.H = H;
  ap.g = cu_seqlens ? g : 1;
  ap.top_k = top_k;
  ap.scale = 1.0f / sqrtf(static_cast<float>(d));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    TraceScope tr("sparse_attention", st);
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(R) * H);
    if (d == 128)
      sparse_attention_kernel<128><<<grid, kAttNT, 0, st>>>(ap);
    else
      sparse_attention_kernel<64><<<grid, kAttNT, 0, st>>>(ap);
  }
  CUDA_TRY(cudaGetLastError());
  return PIVOT_OK;
}

int pivot_decode_index_paged(const void* q, const void* kpages, const int32_t* block_table, const int32_t* seqlens,
                             int B, int H, int d, int g, int page_size, int max_pages, int top_k, int Kc, int mode,
                             int max_seqlen, int32_t* out_idx, float* out_scores, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (page_size < 1 || (page_size & (page_size - 1)) != 0)
    return fail(PIVOT_ERR_INVALID_ARG, "page_size must be a power of two (got %d)", page_size);
  int log2_page = 0;
  while ((1 << log2_page) < page_size) ++log2_page;
  const CacheIndex ci{nullptr, seqlens, block_table, max_pages, log2_page};
  return run_decode(q, kpages, ci, B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, out_scores, nullptr, nullptr,
                    workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pivot_decode_index_ex(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d, int g,
                          int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx, float* out_scores,
                          float* out_proxy, int32_t* out_cand, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return run_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, out_scores, out_proxy,
                    out_cand, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pivot_decode_index(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d, int g,
                       int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx, void* stream) {
  if (int rc = check_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, nullptr))
    return rc;
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = decode_ws_size(B, H, d, g, Kc, mode, max_seqlen);
  return with_temp_workspace(bytes, st, [&](void* ws, size_t n) {
    return run_decode(q, kcache, packed(cu_seqlens), B, H, d, g, top_k, Kc, mode, max_seqlen, out_idx, nullptr, nullptr,
                      nullptr, ws, n, st);
  });
}

int pivot_sync_status(void* stream, int* flags) {
  DeviceInfo* dev = nullptr;
  if (int rc = device_info(&dev)) return rc;
  CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  CUDA_TRY(cudaMemcpy(&v, dev->status, sizeof v, cudaMemcpyDeviceToHost));
  const int zero = 0;
  CUDA_TRY(cudaMemcpy(dev->status, &zero, sizeof zero, cudaMemcpyHostToDevice));
  if (flags) *flags = v;
  if (v & kStTimeout) return fail(PIVOT_ERR_TIMEOUT, "a kernel wait timed out; outputs of that call are invalid");
  if (v & kStBadLen) return fail(PIVOT_ERR_INVALID_ARG, "a decode sequence was longer than max_seqlen");
  if (v & kStNoConverge) return fail(PIVOT_ERR_CUDA, "a refine selection did not converge; outputs of that call are invalid");
  return PIVOT_OK;
}

const char* pivot_last_error(void) { return g_err; }

int pivot_set_wait_limit(unsigned long long ns) {
  g_wait_ns.store(ns);
  return PIVOT_OK;
}

int pivot_trace_enable(int on) {
  g_trace_on = on != 0;
  return PIVOT_OK;
}

int pivot_trace_collect(char* names, size_t names_len, float* ms, int* count, int max_items) {
  // Aggregate by kernel name: ms[i] = total time, count[i] = launches.
  std::vector<const char*> keys;
  std::vector<double> tot;
  std::vector<int> cnt;
  int rc = PIVOT_OK;
  for (TraceRec& r : g_trace) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      rc = fail(PIVOT_ERR_CUDA, "trace event query failed");
    size_t i = 0;
    while (i < keys.size() && strcmp(keys[i], r.name) != 0) ++i;
    if (i == keys.size()) {
      keys.push_back(r.name);
      tot.push_back(0.0);
      cnt.push_back(0);
    }
    tot[i] += t;
    cnt[i] += 1;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_trace.clear();
  size_t off = 0;
  if (names && names_len) names[0] = 0;
  const int n = static_cast<int>(std::min<size_t>(keys.size(), max_items > 0 ? max_items : 0));
  for (int i = 0; i < n; ++i) {
    if (ms) ms[i] = static_cast<float>(tot[i]);
    if (count) count[i] = cnt[i];
    if (names) {
      const int w = snprintf(names + off, off < names_len ? names_len - off : 0, "%s%s", i ? "," : "", keys[i]);
      off += w > 0 ? static_cast<size_t>(w) : 0;
    }
  }
  return rc == PIVOT_OK ? n : -rc;
}

}  // extern "C"
