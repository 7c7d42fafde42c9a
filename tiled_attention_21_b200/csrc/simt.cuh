// simt.cuh -- exact attention forward on the CUDA cores.
//
// The fp32 path (and the decode shapes the tensor-core kernels do not
// cover): FFMA dot products, warp-shuffle row reductions, an online softmax
// in the exp2 domain with the scale folded into scale*log2(e)
// (kernelbot-amd-mixed-mla 588924: SM_SCALE_LOG2E; oxillama-runtime 0.1.0
// flash_attention.rs, flash_attention: tile max, correction factor, running
// sum, normalise once at the end).
//
// Work split: a block of kSimtWarps warps serves kSimtWarps "rows" of one
// (sequence, kv head); row r of the block is query token r / G and q head
// g*G + r % G, so all of them read the same K/V tiles (the row flattening
// of kernelbot-amd-mixed-mla 588924, _flash_fused: m = q_idx*heads + head).
// One warp owns one row.  Keys are processed in tiles of 32, staged in
// shared memory as fp32 (K rows padded by one word so the 32 lanes, one key
// each, hit 32 different banks).  Lane l scores key l of the tile; for P.V
// lane l owns output columns l, l+32, ...
#pragma once

#include "common.cuh"

namespace mxfa {

constexpr int kSimtWarps = 8;
constexpr int kSimtKeys = 32;
constexpr int kSimtStage = 8;  // loads in flight per thread while a tile is staged


__host__ __device__ inline size_t simt_smem_bytes(int dqk, int dv) {
  return sizeof(float) * ((size_t)kSimtWarps * dqk + (size_t)kSimtKeys * (dqk + 1) + (size_t)kSimtKeys * dv);
}

template <typename T, int DV_PER_LANE>
__global__ void __launch_bounds__(kSimtWarps * 32, 2)
attn_fwd_simt_kernel(const AttnParams p) {
  extern __shared__ float smem[];
  const int dqk = p.dqk, dv = p.dv;
  float *qs = smem;                                   // [kSimtWarps][dqk]
  float *ks = qs + kSimtWarps * dqk;                  // [kSimtKeys][dqk + 1]
  float *vs = ks + kSimtKeys * (dqk + 1);             // [kSimtKeys][dv]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y;
  const SeqRange sr = seq_range(p, b);
  const int G = p.hq / p.hkv;
  const int row = blockIdx.x * kSimtWarps + warp;    // flattened (query, head-in-group)
  const int n_rows = sr.sq * G;
  if (blockIdx.x * kSimtWarps >= n_rows) return;     // whole block idle (uniform)

  const bool active = row < n_rows;
  const int i = active ? row / G : 0;
  const int h = g * G + (active ? row % G : 0);
  const int n_vis = active ? visible_keys(i, sr.sq, sr.sk, p.causal) : 0;

  // Keys the block needs: the largest visible count over its rows.
  const int last_row = min(n_rows, (int)(blockIdx.x + 1) * kSimtWarps) - 1;
  const int block_keys = visible_keys(last_row / G, sr.sq, sr.sk, p.causal);

  const T *qrow = reinterpret_cast<const T *>(p.q) + (int64_t)(sr.q0 + i) * p.q_rs + (int64_t)h * p.q_hs;
  for (int d = lane; d < dqk; d += 32) qs[warp * dqk + d] = active ? to_f32(qrow[d]) : 0.f;

  float m = -INFINITY, l = 0.f;
  float acc[DV_PER_LANE], acc2[DV_PER_LANE];
#pragma unroll
  for (int e = 0; e < DV_PER_LANE; ++e) acc[e] = acc2[e] = 0.f;

  const T *kbase = reinterpret_cast<const T *>(p.k) + (int64_t)g * p.k_hs;
  const T *vbase = reinterpret_cast<const T *>(p.v) + (int64_t)g * p.v_hs;

  // K and V tiles are staged in 16-byte pieces: a thread issues a batch of
  // independent loads before it converts and stores any of them, so a tile
  // costs about one memory latency.  Rows are 16-byte aligned (the entry
  // points check the pointers and strides), and dqk, dv are multiples of the
  // eight or four elements of a piece.
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kBatch = kSimtStage * kSimtWarps * 32;
  const int kq = dqk / kVec, vq = dv / kVec;
  const int n_pieces = kSimtKeys * (kq + vq);
  // c / kq and c / vq as a multiply-high by ceil(2^32 / divisor): exact for
  // c * divisor^2 < 2^32 (here c < 32 * 288 and divisors <= 144)
  const uint32_t mk = (uint32_t)(((1ull << 32) + kq - 1) / kq), mv = (uint32_t)(((1ull << 32) + vq - 1) / vq);
  auto load = [&](int t, int base, uint4 (&w)[kSimtStage]) {
    const int nk = min(kSimtKeys, block_keys - t);
#pragma unroll
    for (int u = 0; u < kSimtStage; ++u) {
      const int c = base + u * kSimtWarps * 32;
      w[u] = make_uint4(0, 0, 0, 0);
      if (c < kSimtKeys * kq) {
        const int j = (int)__umulhi((uint32_t)c, mk), dc = c - j * kq;
        if (j < nk) w[u] = *reinterpret_cast<const uint4 *>(kbase + (int64_t)(sr.k0 + t + j) * p.k_rs + dc * kVec);
      } else if (c < n_pieces) {
        const int cv = c - kSimtKeys * kq, j = (int)__umulhi((uint32_t)cv, mv), dc = cv - j * vq;
        if (j < nk) w[u] = *reinterpret_cast<const uint4 *>(vbase + (int64_t)(sr.k0 + t + j) * p.v_rs + dc * kVec);
      }
    }
  };
  auto store = [&](int base, const uint4 (&w)[kSimtStage]) {
#pragma unroll
    for (int u = 0; u < kSimtStage; ++u) {
      const int c = base + u * kSimtWarps * 32;
      const T *e = reinterpret_cast<const T *>(&w[u]);
      if (c < kSimtKeys * kq) {
        const int j = (int)__umulhi((uint32_t)c, mk), dc = c - j * kq;
#pragma unroll
        for (int i = 0; i < kVec; ++i) ks[j * (dqk + 1) + dc * kVec + i] = to_f32(e[i]);
      } else if (c < n_pieces) {
        const int cv = c - kSimtKeys * kq, j = (int)__umulhi((uint32_t)cv, mv), dc = cv - j * vq;
#pragma unroll
        for (int i = 0; i < kVec; ++i) vs[j * dv + dc * kVec + i] = to_f32(e[i]);
      }
    }
  };
  for (int t0 = 0; t0 < block_keys; t0 += kSimtKeys) {
    __syncthreads();  // previous tile fully consumed (also orders the qs writes)
    const int nk = min(kSimtKeys, block_keys - t0);
    for (int base = threadIdx.x; base < n_pieces; base += kBatch) {
      uint4 w[kSimtStage];
      load(t0, base, w);
      store(base, w);
    }
    __syncthreads();
    if (!active || t0 >= n_vis) continue;

    // score of key t0 + lane, in the log2 domain: four partial sums over
    // d mod 4 (dqk is a multiple of 4), so the FMA chain is a quarter as long
    const float *kr = ks + lane * (dqk + 1);
    const float *qr = qs + warp * dqk;
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < dqk; d += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) s4[u] = fmaf(qr[d + u], kr[d + u], s4[u]);
    }
    const float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    float x = (t0 + lane < n_vis) ? s * p.scale_log2 : -INFINITY;

    float tmax = x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    const float m_new = fmaxf(m, tmax);
    const float base = (m_new == -INFINITY) ? 0.f : m_new;   // all-masked guard
    const float alpha = exp2f(m - base);                       // 0 when m = -inf
    const float pj = exp2f(x - base);                          // 0 for masked keys
    float psum = pj;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * alpha + psum;
    m = m_new;
#pragma unroll
    for (int e = 0; e < DV_PER_LANE; ++e) acc[e] *= alpha;
#pragma unroll
    for (int e = 0; e < DV_PER_LANE; ++e) acc2[e] *= alpha;
    // P.V: even and odd keys accumulate separately (two independent chains;
    // keys past nk have pj = 0 and zero-filled V rows)
    for (int j = 0; j < nk; j += 2) {
      const float pa = __shfl_sync(0xffffffffu, pj, j), pb = __shfl_sync(0xffffffffu, pj, j + 1);
      const float *va = vs + j * dv, *vb = va + dv;
#pragma unroll
      for (int e = 0; e < DV_PER_LANE; ++e) {
        const int d = lane + 32 * e;
        if (d < dv) {
          acc[e] = fmaf(pa, va[d], acc[e]);
          acc2[e] = fmaf(pb, vb[d], acc2[e]);
        }
      }
    }
  }
  if (!active) return;

  T *orow = reinterpret_cast<T *>(p.o) + (int64_t)(sr.q0 + i) * p.o_rs + (int64_t)h * p.o_hs;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < DV_PER_LANE; ++e) {
    const int d = lane + 32 * e;
    if (d < dv) orow[d] = from_f32<T>((acc[e] + acc2[e]) * inv);
  }
  if (p.lse && lane == 0) {
    const float lse = l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    p.lse[(int64_t)(sr.q0 + i) * p.hq + h] = lse;
  }
}

}  // namespace mxfa
