// decode_gqa.cuh -- split-KV decode for grouped-query heads on the tensor
// cores (sm_100a).
//
// Shape (the flash_attn_with_kvcache decode of mxflashattn 1.4.0 api.py and
// the q_len = 1 decode bench of AstrAI attn_decode_split_kv_mma.cuh): Hq
// query heads in Hkv groups of Hq/Hkv, one K and one V head per group, head
// dim D in {64, 128}, q_len <= 64.  The decode "sequence" v of the split
// schedule (decode_prep_kernel) is (batch entry b, head group gh): G = Hq /
// heads query heads gh*G .. gh*G+G-1 that read KV head gh / subs, with
// q_len*G <= 64 (subs = 1, one group per KV head, whenever q_len*Hq/Hkv <=
// 64).  Its q_len*G query rows, flattened r = q*G + j for token q and head
// gh*G + j, form the M = 64 side of every MMA (rows past q_len*G are zero and
// never stored).
//
// The K and V heads of each sequence are streamed exactly once: 128-key
// tiles arrive by TMA as D/64 column chunks of K followed by D/64 chunks of
// V (128 keys x 64 columns, 128B swizzle) into a ring of kRingTiles tiles.
//     S   = Q K^T   tcgen05.mma M=64 N=128, D/16 K-steps, A = Q (TMEM), B = K;
//                   the K-steps alternate between two accumulators so
//                   consecutive MMAs do not wait on each other; softmax adds them
//     O  += P V     tcgen05.mma M=64 N=D, 8 K-steps, A = P (shared memory), B = V
// TMEM: O in lanes 0-15 of each sub-partition (columns 0..D-1); in lanes
// 16-31 the two S accumulators (columns 0-255) and Q (columns 256..256+D/2).
// Softmax, the lazy rescale of O, the epilogue, the partials of split
// sequences and the bounded waits are those of the MLA kernel in
// decode_tc.cuh; decode_combine_kernel merges the partials.
#pragma once

#include "decode_tc.cuh"

namespace mxfa {

constexpr int kGqThreads = 256;
constexpr int kGqKeys = 128;                    // keys per KV tile
constexpr int kGqChunkBytes = kGqKeys * 128;    // one 64-column chunk of a tile
constexpr int kGqPBytes = kDcRows * kGqKeys * 2;  // P: two 64-key blocks of 64 rows x 128 B
constexpr int kGqQCol = 256;                    // first TMEM column of Q (lanes 16-31)

template <int D>
struct GqaCfg {
  static constexpr int kChunks = D / 64;           // 64-column chunks of one K or V tile
  static constexpr int kTileChunks = 2 * kChunks;  // K chunks, then V chunks
  static constexpr int kRingTiles = D == 128 ? 3 : 6;
  static constexpr int kSlots = kRingTiles * kTileChunks;
  static constexpr int kSmemBytes = kDcCtrlBytes + kSlots * kGqChunkBytes + kGqPBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct GqaCtrl {
  uint64_t q_ready;
  uint64_t tile_full[12], tile_empty[12];
  uint64_t s_full, s_free, p_full, o_done, o_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(GqaCtrl) <= kDcCtrlBytes, "control block");

template <int D, bool BF16>
__global__ void __launch_bounds__(kGqThreads, 1)
attn_decode_gqa_kernel(const __grid_constant__ AttnParams p, const DecodeSched s,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using Cfg = GqaCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  GqaCtrl *ctrl = reinterpret_cast<GqaCtrl *>(smem_raw);
  const uint32_t tiles_u32 = (smem_u32(smem_raw) + kDcCtrlBytes + 1023u) & ~1023u;
  const uint32_t ring_u32 = tiles_u32;                               // kRingTiles x (K, V) chunks
  const uint32_t p_u32 = ring_u32 + Cfg::kSlots * kGqChunkBytes;     // P: two 64-key blocks
  uint8_t *p_gen = smem_raw + (p_u32 - smem_u32(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &ctrl->abort;
  WsHeader *hdr = p.hdr;
  auto b_tf = [&](int x) { return smem_u32(&ctrl->tile_full[x]); };
  auto b_te = [&](int x) { return smem_u32(&ctrl->tile_empty[x]); };
  const uint32_t b_qr = smem_u32(&ctrl->q_ready), b_sf = smem_u32(&ctrl->s_full), b_sx = smem_u32(&ctrl->s_free);
  const uint32_t b_pf = smem_u32(&ctrl->p_full), b_od = smem_u32(&ctrl->o_done), b_oe = smem_u32(&ctrl->o_empty);
  const int G = p.hq / s.heads;  // query heads per KV head

  if (threadIdx.x == 0) {
    mbar_init(b_qr, 128);
    for (int x = 0; x < Cfg::kRingTiles; ++x) {
      mbar_init(b_tf(x), 1);
      mbar_init(b_te(x), 1);
    }
    mbar_init(b_sf, 1);
    mbar_init(b_sx, 128);
    mbar_init(b_pf, 128);
    mbar_init(b_od, 1);
    mbar_init(b_oe, 128);
    mbar_init(smem_u32(&ctrl->drain), 1);
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  // This CTA's pieces: those whose first tile lies in its tile range (or,
  // in the single-launch schedule, piece blockIdx.x if it exists).
  dc_pdl_wait();  // the schedule kernel's output (a no-op in the single launch)
  int seg_lo, seg_hi;
  if (s.arith_k > 0) {
    seg_lo = blockIdx.x;
    seg_hi = (int)(blockIdx.x % s.arith_k) < dc_seg_cnt(p, s, blockIdx.x / s.arith_k) ? seg_lo + 1 : seg_lo;
  } else {
    const int n_segs = (int)*reinterpret_cast<volatile uint32_t *>(&hdr->n_units);
    const int T = (int)*reinterpret_cast<volatile uint32_t *>(&hdr->n_aux);
    seg_lo = dc_lower_bound(s.segs, n_segs, dc_range_start(blockIdx.x, T, gridDim.x));
    seg_hi = dc_lower_bound(s.segs, n_segs, dc_range_start(blockIdx.x + 1, T, gridDim.x));
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t tc = 0;  // tiles issued by this CTA
      bool ok = true;
      for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
        const int4 sd = dc_seg(p, s, sg);
        const DcSeq sq = dc_seq(p, s, sd.x);
        const int b = sq.b, g = sq.kvh;
        const int len = dc_klen(p, s, b);
        for (int j = sd.y; ok && j < sd.z; ++j, ++tc) {
          const int x = tc % Cfg::kRingTiles;
          if (!wait_bar<kDcColdReport>(b_te(x), ((tc / Cfg::kRingTiles) & 1) ^ 1, abort_flag, hdr, kDSiteSlotEmpty, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(b_tf(x), Cfg::kTileChunks * kGqChunkBytes);
          // A tile is one box of 128 rows when its keys are contiguous rows
          // (packed or dense), else one box per cache page of it (the maps'
          // box height is then the page size, a divisor of 128).
          const int box = (p.cu_k || !s.block_table || s.page_size >= kGqKeys) ? kGqKeys : s.page_size;
          for (int i = 0; i < kGqKeys / box; ++i) {
            const int pos = j * kGqKeys + i * box;
            const int row = pos < len ? dc_krow(p, s, b, pos) : -(1 << 30);
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c) {
              tma_load_3d(ring_u32 + (x * Cfg::kTileChunks + c) * kGqChunkBytes + i * box * 128, &tm_k, b_tf(x), c * 64,
                          g, row);
              tma_load_3d(ring_u32 + (x * Cfg::kTileChunks + Cfg::kChunks + c) * kGqChunkBytes + i * box * 128, &tm_v,
                          b_tf(x), c * 64, g, row);
            }
          }
        }
      }
      // Teardown: every tile load this thread issued must have landed.
      const uint64_t t0 = global_ns();
      for (int x = 0; x < Cfg::kRingTiles; ++x) {
        const uint32_t uses = tc / Cfg::kRingTiles + ((uint32_t)x < tc % Cfg::kRingTiles ? 1u : 0u);
        if (uses == 0) continue;
        while (!mbar_test(b_tf(x), (uses - 1) & 1) && global_ns() - t0 < p.wait_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule (warp-uniform operands); one elected
    // lane issues each tcgen05 operation; the warp gives up a wait together.
    const bool leader = elect_one();
    auto wait_warp = [&](uint32_t bar, uint32_t parity, uint32_t site) {
      return __all_sync(0xffffffffu, wait_bar<kDcColdReport>(bar, parity, abort_flag, hdr, site, p.wait_ns));
    };
    constexpr uint32_t idesc_s = make_idesc_f16(BF16, kDcRows, kGqKeys, false, false);
    constexpr uint32_t idesc_o = make_idesc_f16(BF16, kDcRows, D, false, true);
    const uint32_t tmem_w = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t s_tmem = tmem_w + (16u << 16);  // S accumulators and Q: lanes 16-31 of each sub-partition
    uint32_t tc = 0, g = 0, o_uses = 0;
    bool ok = true;
    const uint32_t k_hi = desc_hi(make_sdesc_sw128(ring_u32, 16, 1024));
    const uint32_t k_lo0 = desc_lo(make_sdesc_sw128(ring_u32, 16, 1024));
    const uint32_t v_hi = desc_hi(make_sdesc_sw128(ring_u32, kGqChunkBytes, 1024));
    const uint32_t v_lo0 = desc_lo(make_sdesc_sw128(ring_u32, kGqChunkBytes, 1024));
    const uint32_t p_hi = desc_hi(make_sdesc_sw128(p_u32, 16, 1024));
    const uint32_t p_lo0 = desc_lo(make_sdesc_sw128(p_u32, 16, 1024));
    // S of tile counter `t`: K-step kk into accumulator kk % 2.
    auto issue_s = [&](uint32_t t) -> bool {
      const int x = t % Cfg::kRingTiles;
      if (!wait_warp(b_tf(x), (t / Cfg::kRingTiles) & 1, kDSiteSlotFull)) return false;
      tc_fence_after();
      const uint32_t k_lo = k_lo0 + (uint32_t)((x * Cfg::kTileChunks * kGqChunkBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        if (leader)
          mma_ts2(s_tmem + (kk & 1) * kGqKeys, s_tmem + kGqQCol + kk * 8,
                  k_lo + (uint32_t)(((kk >> 2) * kGqChunkBytes + (kk & 3) * 32) >> 4), k_hi, idesc_s,
                  kk >= 2 ? 1u : 0u);
      if (leader) mma_commit(b_sf);
      return true;
    };
    for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
      const int4 sd = dc_seg(p, s, sg);
      const int n = sd.z - sd.y;
      if (!wait_warp(b_qr, (sg - seg_lo) & 1, kDSiteQReady)) break;
      tc_fence_after();
      if (g > 0 && !wait_warp(b_sx, (g - 1) & 1, kDSiteSFree)) break;
      if (!issue_s(tc)) break;
      for (int jj = 0; jj < n; ++jj, ++g, ++tc) {
        if (jj + 1 < n) {
          // the single S buffer is free once softmax has read S(g)
          if (!wait_warp(b_sx, g & 1, kDSiteSFree) || !issue_s(tc + 1)) {
            ok = false;
            break;
          }
        }
        if (!wait_warp(b_pf, g & 1, kDSitePFull)) {
          ok = false;
          break;
        }
        if (jj == 0 && o_uses > 0 && !wait_warp(b_oe, (o_uses - 1) & 1, kDSiteOEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t v_lo =
            v_lo0 + (uint32_t)((((tc % Cfg::kRingTiles) * Cfg::kTileChunks + Cfg::kChunks) * kGqChunkBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kGqKeys / 16; ++kk)
          if (leader)
            mma_ss2(tmem_w, p_lo0 + (uint32_t)(((kk >> 2) * (kDcRows * 128) + (kk & 3) * 32) >> 4), p_hi,
                    v_lo + (uint32_t)((kk * 16 * 128) >> 4), v_hi, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        if (leader) {
          mma_commit(b_od);
          mma_commit(b_te(tc % Cfg::kRingTiles));
        }
      }
      ++o_uses;
    }
    if (leader) mma_commit(smem_u32(&ctrl->drain));
    const uint64_t t0 = global_ns();
    while (!mbar_test(smem_u32(&ctrl->drain), 0) && global_ns() - t0 < p.wait_ns) {
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int sub = warp & 3, half = lane >> 4;
    const int r = sub * 16 + (lane & 15);                    // query row of this thread
    const uint32_t o_row = tmem + ((uint32_t)(sub * 32) << 16);
    const uint32_t s_row = tmem + ((uint32_t)(sub * 32 + 16) << 16);
    const float c = p.scale_log2;
    const bool neg = c < 0.f;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    // Q rows of piece sg into TMEM (lanes 16-31, columns kGqQCol..): this
    // thread writes half `half` of row r.
    auto load_q = [&](int sg) {
      const DcSeq ds = dc_seq(p, s, dc_seg(p, s, sg).x);
      const int b = ds.b, gh = ds.gh;
      const int q0 = dc_q(p, b).x, rows = dc_q(p, b).y * G;
      const bool vq = r < rows;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const uint16_t *>(p.q) +
          (vq ? ((int64_t)(q0 + r / G) * p.q_rs + (int64_t)(gh * G + r % G) * p.q_hs + half * (D / 2)) : 0));
      uint32_t w[D / 4];
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        const uint4 u = vq ? src[i] : make_uint4(0, 0, 0, 0);
        w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
      }
      if constexpr (D == 128) tmem_st_half32(s_row + kGqQCol, w);
      else tmem_st_half16(s_row + kGqQCol, w);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_qr);
    };
    uint32_t g = 0;
    bool ok = true;
    if (seg_lo < seg_hi) load_q(seg_lo);
    for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
      const int4 sd = dc_seg(p, s, sg);
      const int v = sd.x;
      const DcSeq ds = dc_seq(p, s, v);
      const int b = ds.b, gh = ds.gh;
      const int q0 = dc_q(p, b).x, sq = dc_q(p, b).y, sk = dc_klen(p, s, b);
      const int rows = sq * G;
      const bool valid = r < rows;
      const int nv = valid ? visible_keys(r / G, sq, sk, p.causal) : 0;
      float m_used = -INFINITY, l = 0.f;
      for (int j = sd.y; j < sd.z; ++j, ++g) {
        const bool got = wait_bar<kDcColdReport>(b_sf, g & 1, abort_flag, hdr, kDSiteSFull, p.wait_ns);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // This thread's 64 keys: block i in {0, 1} holds keys 64i + 32*half + e.
        uint32_t sv[2][32];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint32_t sb[32];
          tmem_ld_half32(s_row + i * 64, sv[i]);
          tmem_ld_half32(s_row + kGqKeys + i * 64, sb);
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[i][e] = __float_as_uint(__uint_as_float(sv[i][e]) + __uint_as_float(sb[e]));
        }
        tc_fence_before();
        mbar_arrive(b_sx);  // S may be overwritten now
        int lim[2];  // keys [0, lim[i]) of block i of this thread are visible
#pragma unroll
        for (int i = 0; i < 2; ++i) lim[i] = nv - j * kGqKeys - i * 64 - half * 32;
        float ext = -INFINITY;
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x = neg ? -__uint_as_float(sv[i][e]) : __uint_as_float(sv[i][e]);
            ext = (e < lim[i]) ? fmaxf(ext, x) : ext;
          }
        ext = fmaxf(ext, __shfl_xor_sync(0xffffffffu, ext, 16));
        const float m_tile = (ext == -INFINITY) ? -INFINITY : (neg ? -ext : ext) * c;
        const float m_new = fmaxf(m_used, m_tile);
        float alpha = 1.f;
        bool need = false;
        if (m_used == -INFINITY) {
          m_used = m_new;
        } else if (m_new > m_used + 8.f) {
          alpha = ex2(m_used - m_new);
          m_used = m_new;
          need = true;
        }
        const float base = (m_used == -INFINITY) ? 0.f : m_used;
        uint32_t pk[2][16];
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = ex2(fmaf(__uint_as_float(sv[i][2 * e]), c, -base));
            float p1 = ex2(fmaf(__uint_as_float(sv[i][2 * e + 1]), c, -base));
            p0 = (2 * e < lim[i]) ? p0 : 0.f;
            p1 = (2 * e + 1 < lim[i]) ? p1 : 0.f;
            rs += p0 + p1;
            pk[i][e] = BF16 ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
          }
        l = l * alpha + rs;
        // P (single buffer) and O may be touched only once the previous P.V is done.
        if (g > 0) {
          const bool got_o = wait_bar<kDcColdReport>(b_od, (g - 1) & 1, abort_flag, hdr, kDSiteODone, p.wait_ns);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got_o)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (j > sd.y && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int q = 0; q < D / 64; ++q) {
            uint32_t ov[32];
            tmem_ld_half32(o_row + q * 64, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st_half32(o_row + q * 64, ov);
          }
          tmem_wait_st();
        }
        // P row r, block i (keys 64i..64i+63, 64 rows x 128 B, 128B swizzle):
        // this thread's keys 32*half.. are four 16-byte chunks of the row.
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint8_t *prow = p_gen + i * (kDcRows * 128) + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (half * 4 + q) ^ (r & 7);
            *reinterpret_cast<uint4 *>(prow + chunk * 16) =
                make_uint4(pk[i][4 * q], pk[i][4 * q + 1], pk[i][4 * q + 2], pk[i][4 * q + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pf);
      }
      if (!ok) break;
      // Every S of this piece has been read, so Q of the next piece may go in.
      if (sg + 1 < seg_hi) load_q(sg + 1);
      // ---------------- epilogue of this piece
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      if (sd.z > sd.y) {
        const bool got_o = wait_bar<kDcColdReport>(b_od, (g - 1) & 1, abort_flag, hdr, kDSiteODone, p.wait_ns);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got_o)) break;
        tc_fence_after();
      }
      const bool direct = dc_seg_cnt(p, s, v) == 1;
      const int tok = q0 + (valid ? r / G : 0), h = gh * G + (valid ? r % G : 0);
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        uint32_t ov[32];
        tmem_ld_half32(o_row + q * 64, ov);
        const int col = q * 64 + half * 32;
        if (!valid) continue;
        if (direct) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = BF16 ? pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv)
                         : pack_f16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
          T *orow = reinterpret_cast<T *>(p.o) + (int64_t)tok * p.o_rs + (int64_t)h * p.o_hs + col;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4 *>(orow)[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *dc_pacc<D>(s, sg, r, col / 4 + e) = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                 __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(b_oe);
      if (valid && half == 0) {
        if (direct) {
          if (p.lse) p.lse[(int64_t)tok * p.hq + h] = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        } else {
          s.part_ml[(int64_t)sg * kDcRows + r] = make_float2(m_used, l);
        }
      }
    }
  }

  dc_pdl_release();  // this CTA's pieces are done: the combine kernel may launch
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (s.arith_k > 0) {
    // single-launch schedule: the pieces of a split sequence merge here (the
    // K/V ring, drained above, is the scratch space)
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const int v = blockIdx.x / s.arith_k, i = blockIdx.x % s.arith_k, k = dc_seg_cnt(p, s, v);
    float *scratch = reinterpret_cast<float *>(smem_raw + kDcCtrlBytes);
    if (k > 1 && i < k) dc_merge_pieces<T, D, kGqThreads>(p, s, v, i, k, scratch);
    else if (k == 0 && i == 0) dc_zero_rows<T, D, kGqThreads>(p, s, v);
  }
}

// ----------------------------------------------------------------------------
// KV-cache append (the k / v arguments of mxflashattn flash_attn_with_kvcache):
// row i of batch entry b of k_new / v_new ([B, snew, Hkv, D]) goes to key
// position cache_seqlens[b] + i of the cache, before the attention reads it.
// Block (i, b); each thread copies 16-byte pieces of the Hkv*D values.  A
// position past the cache's capacity, or a page outside the pool, is not
// written; the call then reports MXFA_ERR_INVALID_ARG in the workspace.
__global__ void __launch_bounds__(256) kv_append_kernel(const AttnParams p, const DecodeSched s, const void *k_new,
                                                         const void *v_new, int snew, int num_rows) {
  const int i = blockIdx.x, b = blockIdx.y;
  const int pos = s.cache_seqlens[b] + i;
  int row;
  if (!s.block_table) {
    row = (pos >= 0 && pos < s.page_size) ? b * s.page_size + pos : -1;
  } else {
    const int idx = pos / s.page_size;
    const int page = (pos >= 0 && idx < s.max_blocks) ? s.block_table[(int64_t)b * s.max_blocks + idx] : -1;
    row = page >= 0 ? page * s.page_size + pos % s.page_size : -1;
  }
  if (row < 0 || row >= num_rows) {
    if (threadIdx.x == 0) report_error_cold(p.hdr, 1u /* MXFA_ERR_INVALID_ARG */, 0x501);
    return;
  }
  const int per_row = p.hkv * p.dqk / 8;  // 16-byte pieces of one token's K (or V)
  const uint4 *ks = reinterpret_cast<const uint4 *>(k_new) + ((int64_t)b * snew + i) * per_row;
  const uint4 *vs = reinterpret_cast<const uint4 *>(v_new) + ((int64_t)b * snew + i) * per_row;
  for (int t = threadIdx.x; t < per_row; t += blockDim.x) {
    const int g = t / (p.dqk / 8), c = t % (p.dqk / 8);
    reinterpret_cast<uint4 *>(const_cast<void *>(p.k))[((int64_t)row * p.k_rs + (int64_t)g * p.k_hs) / 8 + c] = ks[t];
    reinterpret_cast<uint4 *>(const_cast<void *>(p.v))[((int64_t)row * p.v_rs + (int64_t)g * p.v_hs) / 8 + c] = vs[t];
  }
}

}  // namespace mxfa
