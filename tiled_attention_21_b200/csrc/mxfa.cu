// mxfa.cu -- host side of the C ABI declared in include/mxfa.h.
//
// Validates arguments (nothing is launched when a check fails), encodes the
// TMA tensor maps, carves the caller's workspace and enqueues the kernels on
// the caller's stream.  It never allocates device memory and never
// synchronises, except in strict-validation mode and in
// mxfa_read_device_status, which are documented to.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <set>
#include <utility>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "mxfa.h"

#include "common.cuh"
#include "simt.cuh"
#include "prefill_tc.cuh"
#include "sched.cuh"
#include "decode_tc.cuh"
#include "decode_gqa.cuh"

using namespace mxfa;

namespace {

thread_local std::string g_err;
thread_local uint32_t g_detail = 0;

mxfa_status_t fail(mxfa_status_t s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

mxfa_status_t cuda_fail(cudaError_t e, const char *what) {
  return fail(MXFA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MXFA_CUDA(call)                               \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool strict_mode() {
  static int v = [] {
    const char *e = std::getenv("MXFA_STRICT_VALIDATION");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  return v != 0;
}

int elem_bytes(mxfa_dtype_t dt) { return dt == MXFA_F32 ? 4 : 2; }

bool dtype_ok(int dt) { return dt == MXFA_F32 || dt == MXFA_F16 || dt == MXFA_BF16; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- device facts
std::mutex g_dev_mu;
std::vector<int> g_sms;
std::set<std::pair<const void *, int>> g_smem_set;

mxfa_status_t sm_count(int *out) {
  int dev = 0;
  MXFA_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if ((int)g_sms.size() <= dev) g_sms.resize(dev + 1, 0);
  if (g_sms[dev] == 0) MXFA_CUDA(cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev));
  *out = g_sms[dev];
  return MXFA_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
mxfa_status_t ensure_smem(const void *kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return MXFA_OK;
  int dev = 0;
  MXFA_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_smem_set.count({kernel, dev})) return MXFA_OK;
  MXFA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  g_smem_set.insert({kernel, dev});
  return MXFA_OK;
}

// A kernel that moves registers between warpgroups (setmaxnreg) is only
// safe with the per-thread register count its split was computed for.
std::set<const void *> g_regs_ok;
mxfa_status_t check_launch_regs(const void *kernel, int expected) {
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_regs_ok.count(kernel)) return MXFA_OK;
  }
  cudaFuncAttributes a;
  MXFA_CUDA(cudaFuncGetAttributes(&a, kernel));
  if (a.numRegs != expected)
    return fail(MXFA_ERR_UNSUPPORTED, "kernel built with %d registers per thread, its register split needs %d",
                a.numRegs, expected);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  g_regs_ok.insert(kernel);
  return MXFA_OK;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

mxfa_status_t get_encoder(EncodeTiledFn *fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(MXFA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (%s)", cudaGetErrorString(err));
  *fn = cached;
  return MXFA_OK;
}

// 3-D map over [rows][heads][D] (16-bit elements), box = `box_rows` rows x
// 1 head x 64 columns, 128-byte swizzle; rows past `rows` read as zero.
mxfa_status_t make_map(CUtensorMap *map, const void *base, mxfa_dtype_t dt, int D, int heads, int64_t rows,
                       int64_t row_stride, int64_t head_stride, int box_rows = kTcBlockM) {
  EncodeTiledFn enc;
  mxfa_status_t st = get_encoder(&enc);
  if (st != MXFA_OK) return st;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)head_stride * 2, (cuuint64_t)row_stride * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt == MXFA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXFA_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MXFA_OK;
}

// 2-D map over [rows][cols] (16-bit elements, row stride in elements), box =
// 64 rows x 64 columns, 128-byte swizzle; rows past `rows` read as zero.
mxfa_status_t make_map_2d(CUtensorMap *map, const void *base, mxfa_dtype_t dt, int cols, int64_t rows,
                          int64_t row_stride) {
  EncodeTiledFn enc;
  mxfa_status_t st = get_encoder(&enc);
  if (st != MXFA_OK) return st;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt == MXFA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXFA_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (2-D) failed (%d)", (int)r);
  return MXFA_OK;
}

// 2-D map over [rows][cols] bytes (E4M3 codes, row stride in bytes), box =
// 64 rows x 64 bytes, no swizzle; rows past `rows` read as zero.
mxfa_status_t make_map_2d_u8(CUtensorMap *map, const void *base, int cols, int64_t rows, int64_t row_stride) {
  EncodeTiledFn enc;
  mxfa_status_t st = get_encoder(&enc);
  if (st != MXFA_OK) return st;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXFA_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (bytes) failed (%d)", (int)r);
  return MXFA_OK;
}

// ---------------------------------------------------------------- validation
mxfa_status_t check_ptr(const void *p, const char *name, bool allow_null = false) {
  if (!p) return allow_null ? MXFA_OK : fail(MXFA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16) return fail(MXFA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return MXFA_OK;
}

mxfa_status_t check_stride(int64_t s, int eb, const char *name) {
  if (s <= 0) return fail(MXFA_ERR_INVALID_ARG, "%s must be positive", name);
  if ((s * eb) % 16) return fail(MXFA_ERR_INVALID_ARG, "%s (%lld elements) is not a multiple of 16 bytes", name,
                                 (long long)s);
  return MXFA_OK;
}

#define MXFA_TRY(x)                      \
  do {                                   \
    mxfa_status_t s_ = (x);              \
    if (s_ != MXFA_OK) return s_;        \
  } while (0)

mxfa_status_t check_workspace(const void *ws, size_t have, size_t need) {
  if (!ws) return fail(MXFA_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(MXFA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (have < need) return fail(MXFA_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", have, need);
  return MXFA_OK;
}

// Strict mode: copy a cumulative-length array to the host and check it.
mxfa_status_t strict_check_cu(const int32_t *cu, int batch, int total, int max_len, const char *name,
                              cudaStream_t st) {
  std::vector<int32_t> h(batch + 1);
  MXFA_CUDA(cudaMemcpyAsync(h.data(), cu, sizeof(int32_t) * (batch + 1), cudaMemcpyDeviceToHost, st));
  MXFA_CUDA(cudaStreamSynchronize(st));
  if (h[0] != 0) return fail(MXFA_ERR_INVALID_ARG, "%s[0] = %d, expected 0", name, h[0]);
  for (int b = 0; b < batch; ++b) {
    const int len = h[b + 1] - h[b];
    if (len < 0) return fail(MXFA_ERR_INVALID_ARG, "%s decreases at %d", name, b);
    if (len > max_len) return fail(MXFA_ERR_INVALID_ARG, "%s: length %d of sequence %d exceeds the maximum %d", name,
                                   len, b, max_len);
  }
  if (h[batch] != total) return fail(MXFA_ERR_INVALID_ARG, "%s[batch] = %d, expected the total %d", name, h[batch],
                                     total);
  return MXFA_OK;
}

float resolve_scale(float s, int dqk) { return std::isnan(s) ? 1.0f / std::sqrt((float)dqk) : s; }

// Testing hooks (mxfa_test_hooks): the budget of every bounded device wait
// of later launches, and whether the one-launch decode leaves its merge
// counters as the caller prepared them in the workspace instead of zeroing
// them.  Process-wide; the defaults are the production behaviour.
std::atomic<uint64_t> g_wait_ns{kWaitBudgetNs};
std::atomic<int> g_keep_merge_counters{0};

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- launchers
template <typename T, int DVL, int KS>
mxfa_status_t launch_simt_dv(const AttnParams &p, dim3 grid, cudaStream_t st) {
  auto k = attn_fwd_simt_kernel<T, DVL, KS>;
  const size_t smem = simt_smem_bytes(p.dqk, p.dv, KS);
  MXFA_TRY(ensure_smem(reinterpret_cast<const void *>(k), smem));
  k<<<grid, kSimtWarps * 32 * KS, smem, st>>>(p);
  MXFA_CUDA(cudaGetLastError());
  return MXFA_OK;
}

// Four key splits per block when the blocks cover at most half the SMs and
// the keys span more than one tile: a row's tiles are then worked on side by
// side instead of one after another (head dims up to 128, where four staged
// tiles fit in shared memory and 1024 threads in the registers).
template <typename T>
mxfa_status_t launch_simt(const AttnParams &p, int max_rows_per_seq_head, cudaStream_t st) {
  const int G = p.hq / p.hkv;
  dim3 grid((unsigned)((max_rows_per_seq_head * (int64_t)G + kSimtWarps - 1) / kSimtWarps), p.hkv, p.batch);
  if (grid.x == 0) return MXFA_OK;
  int sms = 0;
  MXFA_TRY(sm_count(&sms));
  const int64_t blocks = (int64_t)grid.x * grid.y * grid.z;
  if (2 * blocks <= sms && p.max_sk > kSimtKeys && p.dqk <= 128 && p.dv <= 128)
    return p.dv <= 64 ? launch_simt_dv<T, 2, 4>(p, grid, st) : launch_simt_dv<T, 4, 4>(p, grid, st);
  if (p.dv <= 64) return launch_simt_dv<T, 2, 1>(p, grid, st);
  if (p.dv <= 128) return launch_simt_dv<T, 4, 1>(p, grid, st);
  return launch_simt_dv<T, 16, 1>(p, grid, st);
}

mxfa_status_t launch_simt_any(mxfa_dtype_t dt, const AttnParams &p, int max_rows, cudaStream_t st) {
  if (dt == MXFA_F32) return launch_simt<float>(p, max_rows, st);
  if (dt == MXFA_BF16) return launch_simt<__nv_bfloat16>(p, max_rows, st);
  return launch_simt<__half>(p, max_rows, st);
}

template <int D, bool BF16>
mxfa_status_t launch_tc(AttnParams &p, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        cudaStream_t st) {
  int sms = 0;
  MXFA_TRY(sm_count(&sms));
  // Long causal sequences of one length: units dealt as equal-cost pairs of
  // blocks, heads together (L2 reuse of K/V), when there are at least eight
  // pairs per CTA, so the coarser items still balance.
  const int64_t nblk = ((int64_t)p.sq + kTcUnitRows - 1) / kTcUnitRows;
  p.paired = (p.cu_q == nullptr && p.causal && p.sq == p.sk && nblk % 2 == 0 &&
              (int64_t)p.batch * p.hq * (nblk / 2) >= 8 * (int64_t)sms) ? 1 : 0;
  auto k = attn_fwd_tc_kernel<D, BF16>;
  if (kTcRegsIo != kTcLaunchRegs || kTcRegsSoftmax != kTcLaunchRegs)  // a setmaxnreg split is compiled in
    MXFA_TRY(check_launch_regs(reinterpret_cast<const void *>(k), kTcLaunchRegs));
  MXFA_TRY(ensure_smem(reinterpret_cast<const void *>(k), PrefillCfg<D>::kSmemBytes));
  k<<<sms, kTcThreads, PrefillCfg<D>::kSmemBytes, st>>>(p, mq, mk, mv);
  MXFA_CUDA(cudaGetLastError());
  return MXFA_OK;
}

// Workspace layout of the varlen tensor-core prefill.
struct VarlenWs {
  size_t prefix, bucket, pairs, total;
  int n_buckets, max_pairs;
};
VarlenWs varlen_ws(int batch, int max_sq, int max_sk) {
  VarlenWs w;
  w.n_buckets = 2 * ((max_sk + kTcBlockN - 1) / kTcBlockN) + 1;
  w.max_pairs = batch * ((max_sq + kTcUnitRows - 1) / kTcUnitRows);
  w.prefix = sizeof(WsHeader);
  w.bucket = w.prefix + align256(sizeof(int) * (size_t)(batch + 1));
  w.pairs = w.bucket + align256(sizeof(int) * (size_t)w.n_buckets);
  w.total = w.pairs + align256(sizeof(int2) * (size_t)(w.max_pairs > 0 ? w.max_pairs : 1));
  return w;
}

// Shared by the batched and varlen prefill entry points.
mxfa_status_t prefill(AttnParams &p, mxfa_dtype_t dt, int D, bool varlen, int64_t rows_q, int64_t rows_k,
                      void *ws, cudaStream_t st) {
  const bool tc = dt != MXFA_F32 && (D == 64 || D == 128);
  if (!tc) return launch_simt_any(dt, p, p.max_sq, st);
  if (varlen) {
    const VarlenWs w = varlen_ws(p.batch, p.max_sq, p.max_sk);
    char *base = static_cast<char *>(ws);
    int2 *pairs = reinterpret_cast<int2 *>(base + w.pairs);
    prefill_prep_kernel<<<1, kPrepThreads, 0, st>>>(p, reinterpret_cast<int *>(base + w.prefix),
                                                     reinterpret_cast<int *>(base + w.bucket), w.n_buckets, pairs,
                                                     w.max_pairs);
    MXFA_CUDA(cudaGetLastError());
    p.pairs = pairs;
  }
  CUtensorMap mq, mk, mv;
  MXFA_TRY(make_map(&mq, p.q, dt, D, p.hq, rows_q, p.q_rs, p.q_hs));
  MXFA_TRY(make_map(&mk, p.k, dt, D, p.hkv, rows_k, p.k_rs, p.k_hs));
  MXFA_TRY(make_map(&mv, p.v, dt, D, p.hkv, rows_k, p.v_rs, p.v_hs));
  const bool bf = dt == MXFA_BF16;
  if (D == 128) return bf ? launch_tc<128, true>(p, mq, mk, mv, st) : launch_tc<128, false>(p, mq, mk, mv, st);
  return bf ? launch_tc<64, true>(p, mq, mk, mv, st) : launch_tc<64, false>(p, mq, mk, mv, st);
}

// Launch with programmatic stream serialisation: the kernel's CTAs may start
// while the preceding kernel in the stream still runs; the kernel calls
// dc_pdl_wait() before it reads that kernel's results.
mxfa_status_t launch_dependent(const void *kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  MXFA_CUDA(cudaLaunchKernelExC(&cfg, kernel, args));
  return MXFA_OK;
}

// Workspace layout of the tensor-core decode kernels: `batch` decode
// sequences (batch entries x KV heads that form separate sequences), Dv
// output columns.
struct DecodeWs {
  size_t n_tiles, tile_pre, seg_base, seg_cnt, kv_len, sync, multi, segs, part_ml, part_acc, total;
  int max_segs;
};
DecodeWs decode_ws(int batch, int max_kv_len, int num_splits, int dv, int keys) {
  DecodeWs w;
  const int tiles = (max_kv_len + keys - 1) / keys;
  w.max_segs = num_splits > 0 ? batch * std::max(1, std::min(num_splits, tiles)) : batch + kDcMaxGrid;
  w.n_tiles = sizeof(WsHeader);
  w.tile_pre = w.n_tiles + align256(sizeof(int) * (size_t)batch);
  w.seg_base = w.tile_pre + align256(sizeof(int) * (size_t)(batch + 1));
  w.seg_cnt = w.seg_base + align256(sizeof(int) * (size_t)(batch + 1));
  w.kv_len = w.seg_cnt + align256(sizeof(int) * (size_t)batch);
  w.sync = w.kv_len + align256(sizeof(int) * (size_t)batch);
  w.multi = w.sync + align256(sizeof(int) * (size_t)batch);
  w.segs = w.multi + align256(sizeof(int));
  w.part_ml = w.segs + align256(sizeof(int4) * (size_t)w.max_segs);
  w.part_acc = w.part_ml + align256(sizeof(float2) * (size_t)w.max_segs * kDcRows);
  w.total = w.part_acc + align256(sizeof(float) * (size_t)w.max_segs * kDcRows * dv);
  return w;
}

// Head groups per KV head of the tensor-core decode kernels: the smallest
// divisor d of the G query heads sharing a KV head with max_q_len * G / d
// <= 64 query rows per decode sequence (the M side of their MMAs); 0 when
// there is none (max_q_len > 64).
int head_subgroups(int G, int max_q_len) {
  if (max_q_len <= 0) return 1;
  for (int d = 1; d <= G; ++d)
    if (G % d == 0 && (int64_t)max_q_len * (G / d) <= kDcRows) return d;
  return 0;
}

bool decode_tc_eligible(mxfa_dtype_t dt, int Hq, int Hkv, int Dqk, int Dv, int max_q_len, const void *k,
                        const void *v, int64_t k_rs, int64_t v_rs) {
  return dt != MXFA_F32 && Dqk == kDcDqk && Dv == kDcDv && Hkv == 1 && k == v && k_rs == v_rs &&
         head_subgroups(Hq, max_q_len) > 0;
}

// The grouped-query tensor-core decode: K and V heads of dimension 64 or 128,
// 16-bit, at most 64 queries per sequence, rows TMA-addressable.
bool decode_gqa_eligible(mxfa_dtype_t dt, int Hq, int Hkv, int Dqk, int Dv, int max_q_len, int64_t k_rs,
                         int64_t v_rs) {
  return dt != MXFA_F32 && Dqk == Dv && (Dqk == 64 || Dqk == 128) && head_subgroups(Hq / Hkv, max_q_len) > 0 &&
         (k_rs * 2) % 16 == 0 && (v_rs * 2) % 16 == 0;
}

// Multiplier and shift of div_u for the divisor d >= 1 (d < 1 is taken as 1).
DivU make_divu(int d) {
  d = std::max(d, 1);
  int l = 0;
  while ((1ll << l) < d) ++l;
  DivU q;
  q.sh = 31u + (uint32_t)l;
  q.m = (uint32_t)(((1ull << q.sh) + (uint64_t)d - 1) / (uint64_t)d);
  q.d = d;
  return q;
}

// Split schedule in the workspace for `heads` = Hkv * subs decode sequences
// (head groups) per batch entry.
DecodeSched decode_sched(const AttnParams &p, int heads, int subs, int num_splits, int dv, int keys, void *ws,
                         int sms) {
  const DecodeWs w = decode_ws(p.batch * heads, p.max_sk, num_splits, dv, keys);
  char *base = static_cast<char *>(ws);
  DecodeSched s;
  s.heads = heads;
  s.subs = subs;
  s.by_hkv = make_divu(heads / std::max(subs, 1));
  s.by_bh = make_divu(p.batch * (heads / std::max(subs, 1)));
  s.keys = keys;
  s.n_tiles = reinterpret_cast<int *>(base + w.n_tiles);
  s.tile_pre = reinterpret_cast<int *>(base + w.tile_pre);
  s.seg_base = reinterpret_cast<int *>(base + w.seg_base);
  s.seg_cnt = reinterpret_cast<int *>(base + w.seg_cnt);
  s.segs = reinterpret_cast<int4 *>(base + w.segs);
  s.part_ml = reinterpret_cast<float2 *>(base + w.part_ml);
  s.part_acc = reinterpret_cast<float *>(base + w.part_acc);
  s.kv_len = reinterpret_cast<int *>(base + w.kv_len);
  s.sync = reinterpret_cast<int *>(base + w.sync);
  s.n_multi = reinterpret_cast<int *>(base + w.multi);
  s.arith_k = 0;
  s.o_scale = 1.f;
  s.max_segs = w.max_segs;
  s.num_splits = num_splits;
  // Measured on the batch-128 MLA and batch-64 grouped-query workloads (whole
  // deal 15.6 % longer than the even cut): the MLA kernel's 128 KB partials
  // made the even cut 8 % slower, the grouped-query kernel's 32 KB ones made
  // it 5.5 % faster.
  s.whole_pct = dv == kDcDv ? 120 : 100;
  s.grid = std::min(sms, kDcMaxGrid);
  s.cache_seqlens = nullptr;
  s.add = s.advance = 0;
  s.block_table = nullptr;
  s.max_blocks = s.page_size = 0;
  return s;
}

// `kv_rows`: rows of the K / V tensors; `box`: TMA box height (128, or the
// page size of a paged cache with pages shorter than a tile).
// Blocks of the combine kernel: it walks (sequence, 16-column block) items
// with a grid stride, two blocks per SM of the decode grid at most.
int combine_grid(int n_seq, int dv, int decode_grid) {
  const int64_t items = (int64_t)n_seq * (dv / 16);
  return (int)std::max<int64_t>(1, std::min<int64_t>(items, 2 * (int64_t)decode_grid));
}

template <int D, bool BF16>
mxfa_status_t launch_decode_gqa_t(AttnParams &p, const DecodeSched &s, mxfa_dtype_t dt, int64_t kv_rows, int box,
                                  cudaStream_t st) {
  CUtensorMap mk, mv;
  MXFA_TRY(make_map(&mk, p.k, dt, D, p.hkv, kv_rows, p.k_rs, p.k_hs, box));
  MXFA_TRY(make_map(&mv, p.v, dt, D, p.hkv, kv_rows, p.v_rs, p.v_hs, box));
  auto k = attn_decode_gqa_kernel<D, BF16>;
  // Small problems on packed K/V run in one launch, as for the MLA kernel.
  const int n_seq = p.batch * s.heads, max_tiles = (p.max_sk + kGqKeys - 1) / kGqKeys;
  if (s.num_splits == 0 && p.cu_k && n_seq <= s.grid && (int64_t)n_seq * max_tiles <= 4 * (int64_t)s.grid) {
    DecodeSched sa = s;
    const int t_min = max_tiles > 16 ? 4 : 2;  // tiles per piece at least (merge cost vs chain length)
    sa.arith_k = std::max(1, std::min(s.grid / n_seq, (max_tiles + t_min - 1) / t_min));
    if (sa.arith_k > 1 && !g_keep_merge_counters.load())
      MXFA_CUDA(cudaMemsetAsync(sa.sync, 0, sizeof(int) * (size_t)n_seq, st));
    MXFA_TRY(ensure_smem(reinterpret_cast<const void *>(k), GqaCfg<D>::kSmemBytes));
    void *args[] = {&p, &sa, &mk, &mv};
    MXFA_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(k), dim3(n_seq * sa.arith_k),
                                          dim3(kGqThreads), args, GqaCfg<D>::kSmemBytes, st));
    return MXFA_OK;
  }
  decode_prep_kernel<<<1, 1024, 0, st>>>(p, s);
  MXFA_CUDA(cudaGetLastError());
  MXFA_TRY(ensure_smem(reinterpret_cast<const void *>(k), GqaCfg<D>::kSmemBytes));
  DecodeSched sd = s;
  int ns = n_seq;
  void *args[] = {&p, &sd, &mk, &mv};
  MXFA_TRY(launch_dependent(reinterpret_cast<const void *>(k), dim3(s.grid), dim3(kGqThreads), GqaCfg<D>::kSmemBytes,
                            st, args));
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  void *cargs[] = {&p, &sd, &ns};
  MXFA_TRY(launch_dependent(reinterpret_cast<const void *>(decode_combine_kernel<T, D>),
                            dim3(combine_grid(n_seq, D, s.grid)), dim3(kDcCombineThreads), 0, st, cargs));
  return MXFA_OK;
}

mxfa_status_t launch_decode_gqa(AttnParams &p, const DecodeSched &s, mxfa_dtype_t dt, int64_t kv_rows, int box,
                                cudaStream_t st) {
  const bool bf = dt == MXFA_BF16;
  if (p.dqk == 128)
    return bf ? launch_decode_gqa_t<128, true>(p, s, dt, kv_rows, box, st)
              : launch_decode_gqa_t<128, false>(p, s, dt, kv_rows, box, st);
  return bf ? launch_decode_gqa_t<64, true>(p, s, dt, kv_rows, box, st)
            : launch_decode_gqa_t<64, false>(p, s, dt, kv_rows, box, st);
}

// The MLA tensor-core decode.  kv_fp8: the cache holds E4M3 codes
// (row stride p.k_rs bytes) with dequantisation scale o_scale, and q / o are
// bf16; otherwise it holds `dt` values.
mxfa_status_t launch_decode_tc(AttnParams &p, mxfa_dtype_t dt, int total_q, int total_kv, int num_splits, void *ws,
                               cudaStream_t st, bool kv_fp8 = false, float o_scale = 1.f) {
  int sms = 0;
  MXFA_TRY(sm_count(&sms));
  const int subs = head_subgroups(p.hq, p.max_sq);
  DecodeSched s = decode_sched(p, subs, subs, num_splits, kDcDv, kDcKeys, ws, sms);
  s.o_scale = o_scale;
  const int n_seq = p.batch * subs;  // decode sequences: (batch entry, head group)
  CUtensorMap mq, mkv;
  MXFA_TRY(make_map_2d(&mq, p.q, dt, kDcDqk, (int64_t)total_q * p.hq, kDcDqk));
  if (kv_fp8)
    MXFA_TRY(make_map_2d_u8(&mkv, p.k, kDcDqk, total_kv, p.k_rs));
  else
    MXFA_TRY(make_map_2d(&mkv, p.k, dt, kDcDqk, total_kv, p.k_rs));
  const void *k = kv_fp8 ? reinterpret_cast<const void *>(attn_decode_tc_kernel<true, true>)
                  : dt == MXFA_BF16 ? reinterpret_cast<const void *>(attn_decode_tc_kernel<true>)
                                    : reinterpret_cast<const void *>(attn_decode_tc_kernel<false>);
  MXFA_TRY(ensure_smem(k, kDcSmemBytes));
  const int threads = kv_fp8 ? kDcThreadsFp8 : kDcThreads;
  // Small problems run in one launch: no prep kernel (the pieces follow from
  // kv_indptr) and no combine kernel (split sequences merge in the kernel).
  const int max_tiles = (p.max_sk + kDcKeys - 1) / kDcKeys;
  if (num_splits == 0 && n_seq <= s.grid && (int64_t)n_seq * max_tiles <= 4 * (int64_t)s.grid) {
    DecodeSched sa = s;
    const int t_min = max_tiles > 32 ? 4 : 2;  // tiles per piece at least (merge cost vs chain length)
    sa.arith_k = std::max(1, std::min(s.grid / n_seq, (max_tiles + t_min - 1) / t_min));
    if (sa.arith_k > 1 && !g_keep_merge_counters.load())
      MXFA_CUDA(cudaMemsetAsync(sa.sync, 0, sizeof(int) * (size_t)n_seq, st));
    void *args[] = {&p, &sa, &mq, &mkv};
    MXFA_CUDA(cudaLaunchCooperativeKernel(k, dim3(n_seq * sa.arith_k), dim3(threads), args, kDcSmemBytes, st));
    return MXFA_OK;
  }
  decode_prep_kernel<<<1, 1024, 0, st>>>(p, s);
  MXFA_CUDA(cudaGetLastError());
  void *args[] = {&p, &s, &mq, &mkv};
  MXFA_TRY(launch_dependent(k, dim3(s.grid), dim3(threads), kDcSmemBytes, st, args));
  const int cg = combine_grid(n_seq, kDcDv, s.grid);
  int ns = n_seq;
  void *cargs[] = {&p, &s, &ns};
  const void *ck = dt == MXFA_BF16 ? reinterpret_cast<const void *>(decode_combine_kernel<__nv_bfloat16, kDcDv>)
                                   : reinterpret_cast<const void *>(decode_combine_kernel<__half, kDcDv>);
  MXFA_TRY(launch_dependent(ck, dim3(cg), dim3(kDcCombineThreads), 0, st, cargs));
  return MXFA_OK;
}

mxfa_status_t check_heads(int Hq, int Hkv) {
  if (Hq <= 0 || Hkv <= 0) return fail(MXFA_ERR_INVALID_ARG, "head counts must be positive (Hq=%d, Hkv=%d)", Hq, Hkv);
  if (Hq % Hkv) return fail(MXFA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  return MXFA_OK;
}

// ---------------------------------------------------------------- varlen forward
// The arguments of mxfa_attn_varlen_fwd, checked and launched in steps so
// that the entry point with a caller workspace and the one with the
// library's scratch array run the same checks before either touches device
// memory.
struct VarlenArgs {
  const void *q, *k, *v;
  void *o;
  float *lse;
  const int32_t *cu_q, *cu_k;
  int batch, total_q, total_k, max_q, max_k, Hq, Hkv, D;
  mxfa_dtype_t dtype;
  float scale;
  int causal;
};

// Host-side checks; *noop is set for an empty problem (nothing to launch).
mxfa_status_t varlen_check(const VarlenArgs &a, bool *noop) {
  *noop = false;
  if (!dtype_ok(a.dtype)) return fail(MXFA_ERR_INVALID_ARG, "unknown dtype %d", (int)a.dtype);
  if (a.batch < 0 || a.total_q < 0 || a.total_k < 0 || a.max_q < 0 || a.max_k < 0)
    return fail(MXFA_ERR_INVALID_ARG, "negative size");
  MXFA_TRY(check_heads(a.Hq, a.Hkv));
  if (a.D != 64 && a.D != 128) return fail(MXFA_ERR_UNSUPPORTED, "head dim %d is not supported (64 or 128)", a.D);
  if (std::isinf(a.scale)) return fail(MXFA_ERR_INVALID_ARG, "softmax_scale is infinite");
  if (a.batch == 0 || a.total_q == 0) {
    *noop = true;
    return MXFA_OK;
  }
  if (!a.cu_q || !a.cu_k) return fail(MXFA_ERR_INVALID_ARG, "cu_seqlens_q / cu_seqlens_k is NULL");
  if (a.max_q > a.total_q || a.max_k > a.total_k)
    return fail(MXFA_ERR_INVALID_ARG, "max_seqlen exceeds the total token count");
  MXFA_TRY(check_ptr(a.q, "q"));
  MXFA_TRY(check_ptr(a.o, "o"));
  MXFA_TRY(check_ptr(a.lse, "lse", true));
  if (a.total_k > 0) {
    MXFA_TRY(check_ptr(a.k, "k"));
    MXFA_TRY(check_ptr(a.v, "v"));
  }
  return MXFA_OK;
}

// Strict mode: the cumulative lengths checked on the host (synchronises).
mxfa_status_t varlen_strict(const VarlenArgs &a, cudaStream_t st) {
  if (!strict_mode()) return MXFA_OK;
  MXFA_TRY(strict_check_cu(a.cu_q, a.batch, a.total_q, a.max_q, "cu_seqlens_q", st));
  return strict_check_cu(a.cu_k, a.batch, a.total_k, a.max_k, "cu_seqlens_k", st);
}

mxfa_status_t varlen_launch(const VarlenArgs &a, void *workspace, cudaStream_t st) {
  AttnParams p{};
  p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.o; p.lse = a.lse;
  p.cu_q = a.cu_q; p.cu_k = a.cu_k;
  p.batch = a.batch; p.sq = 0; p.sk = 0; p.max_sq = a.max_q; p.max_sk = a.max_k;
  p.hq = a.Hq; p.hkv = a.Hkv; p.dqk = a.D; p.dv = a.D;
  p.q_rs = (int64_t)a.Hq * a.D; p.q_hs = a.D; p.k_rs = (int64_t)a.Hkv * a.D; p.k_hs = a.D;
  p.v_rs = (int64_t)a.Hkv * a.D; p.v_hs = a.D; p.o_rs = (int64_t)a.Hq * a.D; p.o_hs = a.D;
  p.scale_log2 = resolve_scale(a.scale, a.D) * kLog2e;
  p.causal = a.causal ? 1 : 0;
  p.hdr = static_cast<WsHeader *>(workspace);
  p.pairs = nullptr;
  p.wait_ns = g_wait_ns.load();
  return prefill(p, a.dtype, a.D, true, a.total_q, a.total_k, workspace, st);
}

}  // namespace

extern "C" {

const char *mxfa_last_error(void) { return g_err.c_str(); }

uint32_t mxfa_version(void) { return (0u << 16) | (1u << 8) | 0u; }

void mxfa_test_hooks(uint64_t wait_budget_ns, int keep_merge_counters) {
  g_wait_ns.store(wait_budget_ns ? wait_budget_ns : kWaitBudgetNs);
  g_keep_merge_counters.store(keep_merge_counters ? 1 : 0);
}

uint32_t mxfa_device_status_detail(void) { return g_detail; }

mxfa_status_t mxfa_read_device_status(const void *workspace, void *stream) {
  if (!workspace) return fail(MXFA_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  MXFA_CUDA(cudaMemcpyAsync(h, workspace, sizeof h, cudaMemcpyDeviceToHost, st));
  MXFA_CUDA(cudaStreamSynchronize(st));
  g_detail = h[1];
  if (h[0] != 0) {
    MXFA_CUDA(cudaMemsetAsync(const_cast<void *>(workspace), 0, sizeof h, st));
    MXFA_CUDA(cudaStreamSynchronize(st));
    return fail(static_cast<mxfa_status_t>(h[0]), "device reported status %u at site 0x%x", h[0], h[1]);
  }
  return MXFA_OK;
}

size_t mxfa_attn_fwd_workspace_size(int, int, int, int, int, int, mxfa_dtype_t) { return sizeof(WsHeader); }

size_t mxfa_attn_varlen_fwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int, int D,
                                           mxfa_dtype_t dtype) {
  if (dtype == MXFA_F32 || (D != 64 && D != 128) || batch <= 0) return sizeof(WsHeader);
  return varlen_ws(batch, max_seqlen_q, max_seqlen_k).total;
}

mxfa_status_t mxfa_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Sq, int Sk,
                            int Hq, int Hkv, int D, mxfa_dtype_t dtype, int64_t q_row_stride, int64_t q_head_stride,
                            int64_t k_row_stride, int64_t k_head_stride, int64_t v_row_stride,
                            int64_t v_head_stride, int64_t o_row_stride, int64_t o_head_stride, float softmax_scale,
                            int causal, void *workspace, size_t workspace_bytes, void *stream) {
  if (!dtype_ok(dtype)) return fail(MXFA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (B < 0 || Sq < 0 || Sk < 0) return fail(MXFA_ERR_INVALID_ARG, "negative size (B=%d, Sq=%d, Sk=%d)", B, Sq, Sk);
  MXFA_TRY(check_heads(Hq, Hkv));
  if (D != 64 && D != 128) return fail(MXFA_ERR_UNSUPPORTED, "head dim %d is not supported (64 or 128)", D);
  if (std::isinf(softmax_scale)) return fail(MXFA_ERR_INVALID_ARG, "softmax_scale is infinite");
  if (B == 0 || Sq == 0) return MXFA_OK;
  const int eb = elem_bytes(dtype);
  MXFA_TRY(check_ptr(q, "q"));
  MXFA_TRY(check_ptr(o, "o"));
  MXFA_TRY(check_ptr(lse, "lse", true));
  if (Sk > 0) {
    MXFA_TRY(check_ptr(k, "k"));
    MXFA_TRY(check_ptr(v, "v"));
  }
  MXFA_TRY(check_stride(q_row_stride, eb, "q_row_stride"));
  MXFA_TRY(check_stride(q_head_stride, eb, "q_head_stride"));
  MXFA_TRY(check_stride(k_row_stride, eb, "k_row_stride"));
  MXFA_TRY(check_stride(k_head_stride, eb, "k_head_stride"));
  MXFA_TRY(check_stride(v_row_stride, eb, "v_row_stride"));
  MXFA_TRY(check_stride(v_head_stride, eb, "v_head_stride"));
  MXFA_TRY(check_stride(o_row_stride, eb, "o_row_stride"));
  MXFA_TRY(check_stride(o_head_stride, eb, "o_head_stride"));
  const int64_t rows_q = (int64_t)B * Sq, rows_k = (int64_t)B * Sk;
  if (rows_q > INT32_MAX || rows_k > INT32_MAX) return fail(MXFA_ERR_INVALID_ARG, "B*S exceeds 2^31 rows");
  MXFA_TRY(check_workspace(workspace, workspace_bytes, mxfa_attn_fwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, dtype)));

  AttnParams p{};
  p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
  p.cu_q = nullptr; p.cu_k = nullptr;
  p.batch = B; p.sq = Sq; p.sk = Sk; p.max_sq = Sq; p.max_sk = Sk;
  p.hq = Hq; p.hkv = Hkv; p.dqk = D; p.dv = D;
  p.q_rs = q_row_stride; p.q_hs = q_head_stride; p.k_rs = k_row_stride; p.k_hs = k_head_stride;
  p.v_rs = v_row_stride; p.v_hs = v_head_stride; p.o_rs = o_row_stride; p.o_hs = o_head_stride;
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.causal = causal ? 1 : 0;
  p.hdr = static_cast<WsHeader *>(workspace);
  p.pairs = nullptr;
  p.wait_ns = g_wait_ns.load();
  return prefill(p, dtype, D, false, rows_q, rows_k, workspace, static_cast<cudaStream_t>(stream));
}

mxfa_status_t mxfa_attn_varlen_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch, int total_q,
                                   int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int D,
                                   mxfa_dtype_t dtype, float softmax_scale, int causal, void *workspace,
                                   size_t workspace_bytes, void *stream) {
  const VarlenArgs a{q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                     max_seqlen_k, Hq, Hkv, D, dtype, softmax_scale, causal};
  bool noop = false;
  MXFA_TRY(varlen_check(a, &noop));
  if (noop) return MXFA_OK;
  MXFA_TRY(check_workspace(workspace, workspace_bytes,
                           mxfa_attn_varlen_fwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, Hq, D, dtype)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MXFA_TRY(varlen_strict(a, st));
  return varlen_launch(a, workspace, st);
}

size_t mxfa_attn_decode_splitkv_workspace_size(int batch, int max_q_len, int Hq, int Hkv, int Dv, int max_kv_len,
                                               int num_splits, mxfa_dtype_t dtype) {
  if (dtype == MXFA_F32 || batch <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || num_splits < 0) return sizeof(WsHeader);
  const int subs = head_subgroups(Hq / Hkv, max_q_len);
  if (Dv == kDcDv && Hkv == 1 && subs > 0)  // MLA
    return decode_ws(batch * subs, max_kv_len, num_splits, kDcDv, kDcKeys).total;
  if ((Dv == 64 || Dv == 128) && subs > 0)  // grouped-query heads
    return decode_ws(batch * Hkv * subs, max_kv_len, num_splits, Dv, kGqKeys).total;
  return sizeof(WsHeader);
}

mxfa_status_t mxfa_attn_decode_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                                       const int32_t *qo_indptr, const int32_t *kv_indptr, int batch, int total_q,
                                       int total_kv, int max_q_len, int max_kv_len, int Hq, int Hkv, int Dqk, int Dv,
                                       int64_t k_row_stride, int64_t v_row_stride, mxfa_dtype_t dtype,
                                       float softmax_scale, int causal, int num_splits, void *workspace,
                                       size_t workspace_bytes, void *stream) {
  if (!dtype_ok(dtype)) return fail(MXFA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (batch < 0 || total_q < 0 || total_kv < 0 || max_q_len < 0 || max_kv_len < 0 || num_splits < 0)
    return fail(MXFA_ERR_INVALID_ARG, "negative size");
  MXFA_TRY(check_heads(Hq, Hkv));
  const bool dims_ok = (Dqk == 64 && Dv == 64) || (Dqk == 128 && Dv == 128) || (Dqk == 576 && Dv == 512);
  if (!dims_ok) return fail(MXFA_ERR_UNSUPPORTED, "(Dqk, Dv) = (%d, %d) is not supported", Dqk, Dv);
  if (std::isinf(softmax_scale)) return fail(MXFA_ERR_INVALID_ARG, "softmax_scale is infinite");
  if (batch == 0 || total_q == 0) return MXFA_OK;
  if (!qo_indptr || !kv_indptr) return fail(MXFA_ERR_INVALID_ARG, "qo_indptr / kv_indptr is NULL");
  if (max_q_len > total_q || max_kv_len > total_kv)
    return fail(MXFA_ERR_INVALID_ARG, "max length exceeds the total count");
  const int eb = elem_bytes(dtype);
  MXFA_TRY(check_ptr(q, "q"));
  MXFA_TRY(check_ptr(o, "o"));
  MXFA_TRY(check_ptr(lse, "lse", true));
  if (total_kv > 0) {
    MXFA_TRY(check_ptr(k, "k"));
    MXFA_TRY(check_ptr(v, "v"));
    MXFA_TRY(check_stride(k_row_stride, eb, "k_row_stride"));
    MXFA_TRY(check_stride(v_row_stride, eb, "v_row_stride"));
    if (k_row_stride < (int64_t)Hkv * Dqk || v_row_stride < (int64_t)Hkv * Dv)
      return fail(MXFA_ERR_INVALID_ARG, "row strides smaller than a row");
  }
  MXFA_TRY(check_workspace(workspace, workspace_bytes,
                           mxfa_attn_decode_splitkv_workspace_size(batch, max_q_len, Hq, Hkv, Dv, max_kv_len,
                                                                   num_splits, dtype)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (strict_mode()) {
    MXFA_TRY(strict_check_cu(qo_indptr, batch, total_q, max_q_len, "qo_indptr", st));
    MXFA_TRY(strict_check_cu(kv_indptr, batch, total_kv, max_kv_len, "kv_indptr", st));
  }
  AttnParams p{};
  p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
  p.cu_q = qo_indptr; p.cu_k = kv_indptr;
  p.batch = batch; p.max_sq = max_q_len; p.max_sk = max_kv_len;
  p.hq = Hq; p.hkv = Hkv; p.dqk = Dqk; p.dv = Dv;
  p.q_rs = (int64_t)Hq * Dqk; p.q_hs = Dqk; p.k_rs = k_row_stride; p.k_hs = Dqk;
  p.v_rs = v_row_stride; p.v_hs = Dv; p.o_rs = (int64_t)Hq * Dv; p.o_hs = Dv;
  p.scale_log2 = resolve_scale(softmax_scale, Dqk) * kLog2e;
  p.causal = causal ? 1 : 0;
  p.hdr = static_cast<WsHeader *>(workspace);
  p.pairs = nullptr;
  p.wait_ns = g_wait_ns.load();
  if (decode_tc_eligible(dtype, Hq, Hkv, Dqk, Dv, max_q_len, k, v, k_row_stride, v_row_stride) && total_kv > 0)
    return launch_decode_tc(p, dtype, total_q, total_kv, num_splits, workspace, st);
  if (decode_gqa_eligible(dtype, Hq, Hkv, Dqk, Dv, max_q_len, k_row_stride, v_row_stride) && total_kv > 0) {
    int sms = 0;
    MXFA_TRY(sm_count(&sms));
    const int subs = head_subgroups(Hq / Hkv, max_q_len);
    const DecodeSched s = decode_sched(p, Hkv * subs, subs, num_splits, Dv, kGqKeys, workspace, sms);
    return launch_decode_gqa(p, s, dtype, total_kv, kGqKeys, st);
  }
  return launch_simt_any(dtype, p, max_q_len, st);
}

size_t mxfa_attn_decode_mla_fp8kv_workspace_size(int batch, int max_q_len, int Hq, int max_kv_len, int num_splits) {
  const int subs = Hq > 0 ? head_subgroups(Hq, max_q_len) : 0;
  if (batch <= 0 || num_splits < 0 || subs == 0) return sizeof(WsHeader);
  return decode_ws(batch * subs, max_kv_len, num_splits, kDcDv, kDcKeys).total;
}

mxfa_status_t mxfa_attn_decode_mla_fp8kv(const void *q, const void *kv, float kv_scale, void *o, float *lse,
                                         const int32_t *qo_indptr, const int32_t *kv_indptr, int batch, int total_q,
                                         int total_kv, int max_q_len, int max_kv_len, int Hq, int64_t kv_row_stride,
                                         float softmax_scale, int causal, int num_splits, void *workspace,
                                         size_t workspace_bytes, void *stream) {
  if (batch < 0 || total_q < 0 || total_kv < 0 || max_q_len < 0 || max_kv_len < 0 || num_splits < 0)
    return fail(MXFA_ERR_INVALID_ARG, "negative size");
  if (Hq <= 0) return fail(MXFA_ERR_INVALID_ARG, "Hq must be positive (Hq=%d)", Hq);
  if (std::isinf(softmax_scale)) return fail(MXFA_ERR_INVALID_ARG, "softmax_scale is infinite");
  if (!std::isfinite(kv_scale)) return fail(MXFA_ERR_INVALID_ARG, "kv_scale is not finite");
  if (max_q_len > kDcRows)
    return fail(MXFA_ERR_UNSUPPORTED, "max_q_len = %d exceeds %d queries per sequence", max_q_len, kDcRows);
  if (batch == 0 || total_q == 0) return MXFA_OK;
  if (!qo_indptr || !kv_indptr) return fail(MXFA_ERR_INVALID_ARG, "qo_indptr / kv_indptr is NULL");
  if (max_q_len > total_q || max_kv_len > total_kv)
    return fail(MXFA_ERR_INVALID_ARG, "max length exceeds the total count");
  MXFA_TRY(check_ptr(q, "q"));
  MXFA_TRY(check_ptr(o, "o"));
  MXFA_TRY(check_ptr(lse, "lse", true));
  MXFA_TRY(check_ptr(kv, "kv"));
  MXFA_TRY(check_stride(kv_row_stride, 1, "kv_row_stride"));
  if (kv_row_stride < kDcDqk) return fail(MXFA_ERR_INVALID_ARG, "kv_row_stride is smaller than a row (576 bytes)");
  MXFA_TRY(check_workspace(workspace, workspace_bytes,
                           mxfa_attn_decode_mla_fp8kv_workspace_size(batch, max_q_len, Hq, max_kv_len, num_splits)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (strict_mode()) {
    MXFA_TRY(strict_check_cu(qo_indptr, batch, total_q, max_q_len, "qo_indptr", st));
    MXFA_TRY(strict_check_cu(kv_indptr, batch, total_kv, max_kv_len, "kv_indptr", st));
  }
  AttnParams p{};
  p.q = q; p.k = kv; p.v = kv; p.o = o; p.lse = lse;
  p.cu_q = qo_indptr; p.cu_k = kv_indptr;
  p.batch = batch; p.max_sq = max_q_len; p.max_sk = max_kv_len;
  p.hq = Hq; p.hkv = 1; p.dqk = kDcDqk; p.dv = kDcDv;
  p.q_rs = (int64_t)Hq * kDcDqk; p.q_hs = kDcDqk; p.k_rs = kv_row_stride; p.k_hs = kDcDqk;
  p.v_rs = kv_row_stride; p.v_hs = kDcDv; p.o_rs = (int64_t)Hq * kDcDv; p.o_hs = kDcDv;
  // s = softmax_scale * <q, kv_scale * code>: the dequantisation scale joins the score scale
  p.scale_log2 = resolve_scale(softmax_scale, kDcDqk) * kv_scale * kLog2e;
  p.causal = causal ? 1 : 0;
  p.hdr = static_cast<WsHeader *>(workspace);
  p.pairs = nullptr;
  p.wait_ns = g_wait_ns.load();
  return launch_decode_tc(p, MXFA_BF16, total_q, total_kv, num_splits, workspace, st, true, kv_scale);
}

size_t mxfa_attn_decode_kvcache_workspace_size(int batch, int Sq, int Hq, int Hkv, int D, int max_len,
                                               int num_splits, mxfa_dtype_t dtype) {
  if (dtype == MXFA_F32 || batch <= 0 || Sq <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || num_splits < 0 ||
      (D != 64 && D != 128) || Sq > kDcRows || max_len < 0)
    return sizeof(WsHeader);
  return decode_ws(batch * Hkv * head_subgroups(Hq / Hkv, Sq), max_len, num_splits, D, kGqKeys).total;
}

mxfa_status_t mxfa_attn_decode_kvcache(const void *q, void *k_cache, void *v_cache, const void *k_new,
                                       const void *v_new, int32_t *cache_seqlens, const int32_t *block_table,
                                       int batch, int Sq, int Snew, int Hq, int Hkv, int D, int num_pages,
                                       int page_size, int max_blocks_per_seq, int max_len, mxfa_dtype_t dtype,
                                       float softmax_scale, int causal, int num_splits, void *o, float *lse,
                                       void *workspace, size_t workspace_bytes, void *stream) {
  if (!dtype_ok(dtype)) return fail(MXFA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (batch < 0 || Sq < 0 || Snew < 0 || num_pages < 0 || page_size <= 0 || max_len < 0 || num_splits < 0 ||
      max_blocks_per_seq < 0)
    return fail(MXFA_ERR_INVALID_ARG, "negative size or non-positive page size");
  MXFA_TRY(check_heads(Hq, Hkv));
  if (D != 64 && D != 128) return fail(MXFA_ERR_UNSUPPORTED, "head dimension %d is not 64 or 128", D);
  if (std::isinf(softmax_scale)) return fail(MXFA_ERR_INVALID_ARG, "softmax_scale is infinite");
  if (dtype == MXFA_F32) return fail(MXFA_ERR_UNSUPPORTED, "the KV-cache decode takes bf16 or f16");
  if (Sq > kDcRows) return fail(MXFA_ERR_UNSUPPORTED, "Sq = %d exceeds %d queries per sequence", Sq, kDcRows);
  if ((k_new == nullptr) != (v_new == nullptr) || (Snew > 0 && k_new == nullptr))
    return fail(MXFA_ERR_INVALID_ARG, "k_new and v_new go together, and Snew > 0 needs them");
  if (batch == 0 || Sq == 0) return MXFA_OK;
  if (!cache_seqlens) return fail(MXFA_ERR_INVALID_ARG, "cache_seqlens is NULL");
  const bool paged = block_table != nullptr;
  if (paged) {
    const bool pow2 = (page_size & (page_size - 1)) == 0;
    if (!((page_size >= 16 && page_size <= kGqKeys && pow2) || page_size % kGqKeys == 0))
      return fail(MXFA_ERR_UNSUPPORTED, "page size %d: a power of two in [16, 128] or a multiple of 128", page_size);
    if (max_blocks_per_seq <= 0) return fail(MXFA_ERR_INVALID_ARG, "block table with no columns");
  } else if (num_pages != batch) {
    return fail(MXFA_ERR_INVALID_ARG, "a dense cache holds one page of page_size rows per batch entry");
  }
  if ((int64_t)num_pages * page_size >= (1ll << 30))
    return fail(MXFA_ERR_UNSUPPORTED, "cache of %lld rows exceeds 2^30", (long long)num_pages * page_size);
  MXFA_TRY(check_ptr(q, "q"));
  MXFA_TRY(check_ptr(o, "o"));
  MXFA_TRY(check_ptr(k_cache, "k_cache"));
  MXFA_TRY(check_ptr(v_cache, "v_cache"));
  MXFA_TRY(check_ptr(lse, "lse", true));
  if (k_new) {
    MXFA_TRY(check_ptr(k_new, "k_new"));
    MXFA_TRY(check_ptr(v_new, "v_new"));
  }
  MXFA_TRY(check_workspace(workspace, workspace_bytes,
                           mxfa_attn_decode_kvcache_workspace_size(batch, Sq, Hq, Hkv, D, max_len, num_splits, dtype)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p{};
  p.q = q; p.k = k_cache; p.v = v_cache; p.o = o; p.lse = lse;
  p.cu_q = nullptr; p.cu_k = nullptr;
  p.batch = batch; p.max_sq = Sq; p.max_sk = max_len;
  p.hq = Hq; p.hkv = Hkv; p.dqk = D; p.dv = D;
  p.q_rs = (int64_t)Hq * D; p.q_hs = D;
  p.k_rs = p.v_rs = (int64_t)Hkv * D; p.k_hs = p.v_hs = D;
  p.o_rs = (int64_t)Hq * D; p.o_hs = D;
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.causal = causal ? 1 : 0;
  p.hdr = static_cast<WsHeader *>(workspace);
  p.pairs = nullptr;
  p.wait_ns = g_wait_ns.load();
  int sms = 0;
  MXFA_TRY(sm_count(&sms));
  const int subs = head_subgroups(Hq / Hkv, Sq);
  DecodeSched s = decode_sched(p, Hkv * subs, subs, num_splits, D, kGqKeys, workspace, sms);
  s.cache_seqlens = cache_seqlens;
  s.add = Snew;
  s.advance = Snew > 0 ? 1 : 0;
  s.block_table = block_table;
  s.max_blocks = paged ? max_blocks_per_seq : 0;
  s.page_size = page_size;
  const int64_t rows = (int64_t)num_pages * page_size;
  if (Snew > 0) {
    kv_append_kernel<<<dim3(Snew, batch), 256, 0, st>>>(p, s, k_new, v_new, Snew, (int)rows);
    MXFA_CUDA(cudaGetLastError());
  }
  return launch_decode_gqa(p, s, dtype, rows, paged && page_size < kGqKeys ? page_size : kGqKeys, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Varlen forward without a caller workspace.
//
// Some callers have no way to allocate device memory at the point where they
// run attention: engine plugins and services that plan every device byte up
// front and forbid allocation afterwards, or code that holds raw pointers but
// no handle to the framework allocator that owns the device.  This entry point
// serves them: the schedule the varlen path needs lives in a fixed scratch
// array that belongs to the library, so the call allocates nothing.
//
// The array is a file-scope __device__ object: every GPU that loads this
// library holds kNoAllocScratchBytes for it until the process exits.  Its name
// is only a host-side stand-in in host code, so the device address is fetched
// with cudaGetSymbolAddress once per device (with that device current) on the
// first call there, and cached.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};

mxfa_status_t noalloc_scratch(void **out) {
  int dev = 0;
  MXFA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(MXFA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MXFA_OK;
}
}  // namespace

extern "C" mxfa_status_t mxfa_attn_varlen_fwd_noalloc(const void *q, const void *k, const void *v, void *o,
                                                      float *lse, const int32_t *cu_seqlens_q,
                                                      const int32_t *cu_seqlens_k, int batch, int total_q,
                                                      int total_k, int max_seqlen_q, int max_seqlen_k, int Hq,
                                                      int Hkv, int D, mxfa_dtype_t dtype, float softmax_scale,
                                                      int causal, void *stream) {
  const VarlenArgs a{q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                     max_seqlen_k, Hq, Hkv, D, dtype, softmax_scale, causal};
  // Every argument check of mxfa_attn_varlen_fwd runs before the scratch
  // array is touched, so a rejected call writes nothing.
  bool noop = false;
  MXFA_TRY(varlen_check(a, &noop));
  if (noop) return MXFA_OK;
  const size_t need = mxfa_attn_varlen_fwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, Hq, D, dtype);
  if (need > kNoAllocScratchBytes)
    return fail(MXFA_ERR_WORKSPACE,
                "this problem needs %zu bytes of scratch but the no-allocation entry point holds %zu; "
                "call mxfa_attn_varlen_fwd with a workspace instead",
                need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  MXFA_TRY(noalloc_scratch(&scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MXFA_TRY(varlen_strict(a, st));
  // The header (status word, unit count) must start at zero; the schedule
  // tables after it are fully rewritten by every call.
  MXFA_CUDA(cudaMemsetAsync(scratch, 0, sizeof(WsHeader), st));
  return varlen_launch(a, scratch, st);
}

// The status word of the scratch array: what mxfa_read_device_status reads
// from a caller's workspace, read here from the array of the current device.
extern "C" mxfa_status_t mxfa_read_noalloc_status(void *stream) {
  void *scratch = nullptr;
  MXFA_TRY(noalloc_scratch(&scratch));
  return mxfa_read_device_status(scratch, stream);
}
