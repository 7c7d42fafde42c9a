// common.cuh -- shared definitions of the mxfa CUDA kernels (sm_100a).
//
// Parameter block, workspace header, status reporting and the bounded
// wait used by every spin in the library.  PTX wrappers for TMA, mbarrier
// and tcgen05 live in ptx.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace mxfa {

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  uint32_t status;    // 0 = ok, else an mxfa_status_t (first error wins)
  uint32_t detail;    // site code of the first failing wait
  uint32_t n_units;   // number of scheduled work units (written by the prep kernel)
  uint32_t n_aux;     // path-specific count (decode: number of segments)
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr uint32_t kStatusTimeout = 5;  // == MXFA_ERR_TIMEOUT

// Default wait budget of every device-side spin, in nanoseconds of
// %globaltimer; each launch carries its budget in AttnParams::wait_ns.
constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Record the first device-side error; later ones keep the first site.
__device__ __forceinline__ void report_error(WsHeader *hdr, uint32_t code, uint32_t site) {
  if (atomicCAS(&hdr->status, 0u, code) == 0u) atomicExch(&hdr->detail, site);
}
// The same, out of line, for the kernels without a setmaxnreg register split
// (the decode kernels): it runs only when a wait gives up or a schedule
// overflows, and inlined at every bounded wait it made their hot loops longer
// (twice the instruction-cache misses in the grouped-query decode, 4 % of its
// time).  The prefill kernel keeps the inline form, so no call is made from
// a warp whose register budget setmaxnreg has lowered.
__device__ __noinline__ void report_error_cold(WsHeader *hdr, uint32_t code, uint32_t site) {
  report_error(hdr, code, site);
}

// Common parameter block of the attention kernels.  Lengths are either
// uniform (cu_q == nullptr: sequence b holds tokens [b*sq, (b+1)*sq)) or
// read from the int32 cumulative arrays.
struct AttnParams {
  const void *q, *k, *v;
  void *o;
  float *lse;
  const int32_t *cu_q, *cu_k;
  int batch, sq, sk;          // uniform lengths (used when cu_* is null)
  int hq, hkv, dqk, dv;
  int max_sq, max_sk;
  int64_t q_rs, q_hs, k_rs, k_hs, v_rs, v_hs, o_rs, o_hs;  // element strides
  float scale_log2;           // softmax_scale * log2(e)
  int causal;
  WsHeader *hdr;
  const int2 *pairs;          // varlen schedule: sorted (sequence, 256-row block) pairs
  uint64_t wait_ns;           // budget of every bounded device-side wait (kWaitBudgetNs unless a test shortens it)
  int paired;                 // tensor-core prefill: deal units as pairs of 256-row blocks (see unit_at)
};

struct SeqRange {
  int q0, sq, k0, sk;
};

__device__ __forceinline__ SeqRange seq_range(const AttnParams &p, int b) {
  SeqRange r;
  if (p.cu_q) {
    r.q0 = p.cu_q[b];
    r.sq = p.cu_q[b + 1] - r.q0;
  } else {
    r.q0 = b * p.sq;
    r.sq = p.sq;
  }
  if (p.cu_k) {
    r.k0 = p.cu_k[b];
    r.sk = p.cu_k[b + 1] - r.k0;
  } else {
    r.k0 = b * p.sk;
    r.sk = p.sk;
  }
  return r;
}

// Number of keys visible to local query row i (keys 0 .. n-1), from the
// bottom-right causal alignment j <= i + Sk - Sq.
__device__ __forceinline__ int visible_keys(int i, int sq, int sk, int causal) {
  if (!causal) return sk;
  int lim = i + 1 + sk - sq;
  return lim < 0 ? 0 : (lim > sk ? sk : lim);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

}  // namespace mxfa
