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

constexpr int kSimtWarps = 8;   // rows per block
constexpr int kSimtKeys = 32;

// Key splits per block: KS = 1, or 4 for problems with few blocks (the KS
// warps of a row take interleaved 32-key tiles and merge their partial
// (max, sum, accumulator) at the end, so a short sequence is one tile deep
// instead of four).  Loads in flight per thread while tiles are staged.
template <int KS>
constexpr int simt_stage() { return KS == 1 ? 8 : 4; }

__host__ __device__ inline size_t simt_smem_bytes(int dqk, int dv, int ks = 1) {
  const size_t tiles = (size_t)ks * ((size_t)kSimtKeys * (dqk + 1) + (size_t)kSimtKeys * dv);
  const size_t merge = ks > 1 ? (size_t)(ks - 1) * kSimtWarps * (dv + 2) : 0;  // reuses the tile area
  return sizeof(float) * ((size_t)kSimtWarps * dqk + (tiles > merge ? tiles : merge));
}

template <typename T, int DV_PER_LANE, int KS>
__global__ void __launch_bounds__(kSimtWarps * 32 * KS, KS == 1 ? 2 : 1)
attn_fwd_simt_kernel(const AttnParams p) {
  extern __shared__ float smem[];
  const int dqk = p.dqk, dv = p.dv;
  const int tile_floats = kSimtKeys * (dqk + 1) + kSimtKeys * dv;
  float *qs = smem;                                   // [kSimtWarps][dqk]
  float *tiles = qs + kSimtWarps * dqk;               // KS x ([kSimtKeys][dqk + 1], [kSimtKeys][dv])

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rw = warp % kSimtWarps, sp = warp / kSimtWarps;  // row slot, key split
  float *ks = tiles + sp * tile_floats;               // this split's K tile
  float *vs = ks + kSimtKeys * (dqk + 1);             // and V tile
  const int b = blockIdx.z, g = blockIdx.y;
  const SeqRange sr = seq_range(p, b);
  const int G = p.hq / p.hkv;
  const int row = blockIdx.x * kSimtWarps + rw;       // flattened (query, head-in-group)
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
  if (sp == 0)
    for (int d = lane; d < dqk; d += 32) qs[rw * dqk + d] = active ? to_f32(qrow[d]) : 0.f;

  float m = -INFINITY, l = 0.f;
  float acc[DV_PER_LANE], acc2[DV_PER_LANE];
#pragma unroll
  for (int e = 0; e < DV_PER_LANE; ++e) acc[e] = acc2[e] = 0.f;

  const T *kbase = reinterpret_cast<const T *>(p.k) + (int64_t)g * p.k_hs;
  const T *vbase = reinterpret_cast<const T *>(p.v) + (int64_t)g * p.v_hs;

  // K and V tiles are staged in 16-byte pieces: a thread issues a batch of
  // independent loads before it converts and stores any of them, so a group
  // of KS tiles costs about one memory latency.  Rows are 16-byte aligned
  // (the entry points check the pointers and strides), and dqk, dv are
  // multiples of the eight or four elements of a piece.
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kStage = simt_stage<KS>();
  constexpr int kBatch = kStage * kSimtWarps * 32 * KS;
  const int kq = dqk / kVec, vq = dv / kVec;
  const int n_pieces = kSimtKeys * (kq + vq);          // per tile
  // c / kq, c / vq and c / n_pieces as a multiply-high by ceil(2^32 / divisor):
  // exact for c * divisor^2 < 2^32 (here c < KS * n_pieces <= 4 * 32 * 288
  // and divisors <= 144 when KS = 1; c < 4 * 2048, divisors <= 2048 when KS = 4)
  const uint32_t mk = (uint32_t)(((1ull << 32) + kq - 1) / kq), mv = (uint32_t)(((1ull << 32) + vq - 1) / vq);
  const uint32_t mp = (uint32_t)(((1ull << 32) + n_pieces - 1) / n_pieces);
  // piece c of the group: tile s = c / n_pieces, then a K or V row piece
  auto locate = [&](int c, int &s, int &j, int &dc, bool &is_k) {
    s = KS == 1 ? 0 : (int)__umulhi((uint32_t)c, mp);
    const int cl = c - s * n_pieces;
    is_k = cl < kSimtKeys * kq;
    const int cv = is_k ? cl : cl - kSimtKeys * kq;
    j = (int)__umulhi((uint32_t)cv, is_k ? mk : mv);
    dc = cv - j * (is_k ? kq : vq);
  };
  auto load = [&](int t0, int base, uint4 (&w)[kStage]) {
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int c = base + u * kSimtWarps * 32 * KS;
      w[u] = make_uint4(0, 0, 0, 0);
      if (c < KS * n_pieces) {
        int s, j, dc;
        bool is_k;
        locate(c, s, j, dc, is_k);
        const int key = t0 + s * kSimtKeys + j;
        if (key < block_keys && j < kSimtKeys)
          w[u] = is_k ? *reinterpret_cast<const uint4 *>(kbase + (int64_t)(sr.k0 + key) * p.k_rs + dc * kVec)
                      : *reinterpret_cast<const uint4 *>(vbase + (int64_t)(sr.k0 + key) * p.v_rs + dc * kVec);
      }
    }
  };
  auto store = [&](int base, const uint4 (&w)[kStage]) {
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int c = base + u * kSimtWarps * 32 * KS;
      if (c < KS * n_pieces) {
        int s, j, dc;
        bool is_k;
        locate(c, s, j, dc, is_k);
        float *kt = tiles + s * tile_floats, *vt = kt + kSimtKeys * (dqk + 1);
        const T *e = reinterpret_cast<const T *>(&w[u]);
        if (is_k) {
#pragma unroll
          for (int x = 0; x < kVec; ++x) kt[j * (dqk + 1) + dc * kVec + x] = to_f32(e[x]);
        } else {
#pragma unroll
          for (int x = 0; x < kVec; ++x) vt[j * dv + dc * kVec + x] = to_f32(e[x]);
        }
      }
    }
  };
  for (int tg = 0; tg < block_keys; tg += KS * kSimtKeys) {
    __syncthreads();  // previous tiles fully consumed (also orders the qs writes)
    for (int base = threadIdx.x; base < KS * n_pieces; base += kBatch) {
      uint4 w[kStage];
      load(tg, base, w);
      store(base, w);
    }
    __syncthreads();
    const int t0 = tg + sp * kSimtKeys;  // this split's tile
    if (!active || t0 >= n_vis) continue;
    const int nk = min(kSimtKeys, block_keys - t0);

    // score of key t0 + lane, in the log2 domain: four partial sums over
    // d mod 4 (dqk is a multiple of 4), so the FMA chain is a quarter as long
    const float *kr = ks + lane * (dqk + 1);
    const float *qr = qs + rw * dqk;
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < dqk; d += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) s4[u] = fmaf(qr[d + u], kr[d + u], s4[u]);
    }
    const float sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    float x = (t0 + lane < n_vis) ? sc * p.scale_log2 : -INFINITY;

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
#pragma unroll
  for (int e = 0; e < DV_PER_LANE; ++e) acc[e] += acc2[e];

  if constexpr (KS > 1) {
    // Splits 1..KS-1 hand (m, l, acc) to split 0 through the tile area:
    // O = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), M = max_s m_s.
    float *mg = tiles;  // [KS-1][kSimtWarps][dv + 2]
    __syncthreads();    // every split is done with the tiles
    if (active && sp > 0) {
      float *slot = mg + ((sp - 1) * kSimtWarps + rw) * (dv + 2);
      if (lane == 0) {
        slot[dv] = m;
        slot[dv + 1] = l;
      }
#pragma unroll
      for (int e = 0; e < DV_PER_LANE; ++e) {
        const int d = lane + 32 * e;
        if (d < dv) slot[d] = acc[e];
      }
    }
    __syncthreads();
    if (!active || sp > 0) return;
    float M = m;
#pragma unroll
    for (int q = 1; q < KS; ++q) M = fmaxf(M, mg[((q - 1) * kSimtWarps + rw) * (dv + 2) + dv]);
    const float wm = (m == -INFINITY) ? 0.f : exp2f(m - M);  // a split that saw no key weighs 0
    l *= wm;
#pragma unroll
    for (int e = 0; e < DV_PER_LANE; ++e) acc[e] *= wm;
#pragma unroll
    for (int q = 1; q < KS; ++q) {
      const float *slot = mg + ((q - 1) * kSimtWarps + rw) * (dv + 2);
      const float mq = slot[dv];
      const float w = (mq == -INFINITY) ? 0.f : exp2f(mq - M);
      l = fmaf(slot[dv + 1], w, l);
#pragma unroll
      for (int e = 0; e < DV_PER_LANE; ++e) {
        const int d = lane + 32 * e;
        if (d < dv) acc[e] = fmaf(slot[d], w, acc[e]);
      }
    }
    m = M;
  }
  if (!active) return;

  T *orow = reinterpret_cast<T *>(p.o) + (int64_t)(sr.q0 + i) * p.o_rs + (int64_t)h * p.o_hs;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < DV_PER_LANE; ++e) {
    const int d = lane + 32 * e;
    if (d < dv) orow[d] = from_f32<T>(acc[e] * inv);
  }
  if (p.lse && lane == 0) {
    const float lse = l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    p.lse[(int64_t)(sr.q0 + i) * p.hq + h] = lse;
  }
}

}  // namespace mxfa
