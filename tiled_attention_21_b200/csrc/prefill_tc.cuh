// prefill_tc.cuh -- tensor-core attention forward for bf16 / f16 (sm_100a).
//
// One persistent CTA per SM walks a list of work units.  A unit is
// (sequence b, 256-row query block m, query head h) and is processed as two
// 128-row query tiles t = 0, 1 that share every K/V tile.  Per KV tile j
// (128 keys) and query tile t:
//     S_t  = Q_t K_j^T           tcgen05.mma, A = Q (smem), B = K (smem),
//                                fp32 accumulator in TMEM
//     P_t  = exp2(c*S_t - m)     softmax, four threads per row (one per
//                                32-key group g), c = softmax_scale*log2(e);
//                                P written back into TMEM over S_t as
//                                bf16/f16 (keys 32g..32g+31 in columns
//                                32g..32g+15)
//     O_t += P_t V_j             tcgen05.mma, A = P (TMEM), B = V (smem)
// The online-softmax bookkeeping follows mxflashattn 1.4.0 prefill.py
// (prefill_chunked_reference: running max, correction of the accumulator,
// running sum, rows with nothing visible end at O = 0) and oxillama-runtime
// 0.1.0 flash_attention.rs (causal tile skipping), with one change of
// schedule: the accumulator is only rescaled when a row's maximum grows by
// more than 2^8.  Until then O and l keep the stale maximum as their common
// base, which leaves O = acc / l and LSE = base + log2(l) exact.
//
// Roles (768 threads, six warpgroups; launched at 80 registers per thread,
// then setmaxnreg gives warpgroups 0 and 5 48 and warpgroups 1-4 96):
//   warp 0      TMA producer: Q tiles once per unit, then K_j, V_j into a
//               ring of shared-memory slots (128B-swizzled boxes of 64 cols)
//   warp 1      TMEM allocator and MMA issuer: the whole warp runs the
//               schedule and one elected lane issues; it alternates the two
//               query tiles (PV_0(j), S_0(j+1), PV_1(j), S_1(j+1)) so one
//               tile's softmax overlaps the other tile's MMAs
//   warps 2-3   idle (they complete warpgroup 0 for setmaxnreg)
//   warps 4-19  softmax.  A query row has four threads, one per 32-key
//               group g = (warp-4)/4, in the four warps of its TMEM
//               sub-partition (warp w reads lanes 32*(w%4)..+31); these four
//               warps take query tile 0 and query tile 1 in turn, and vote
//               (bar.red.and) on whether the stale base still bounds every
//               row before exchanging partial maxima through shared memory.
//               At the end of a unit they hand the row sums and write LSE.
//   warps 20-23 output epilogue: O_t / l in the output dtype, one thread per
//               row, then O_t's TMEM columns go back to the MMA issuer.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 after it.
//
// Every wait is bounded (see wait_bar_flag); a wait that runs out leaves its
// site in the CTA-wide abort flag, all roles skip to the common teardown,
// which drains the TMA loads and MMAs this CTA issued before TMEM is
// released, and thread 0 records MXFA_ERR_TIMEOUT with that site in the
// workspace.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "exp2_poly.cuh"

namespace mxfa {

constexpr int kTcBlockM = 128;  // rows per query tile
constexpr int kTcBlockN = 128;  // keys per KV tile
constexpr int kTcUnitRows = 2 * kTcBlockM;
constexpr int kTcThreads = 768;
constexpr int kTcSoftmaxThreads = 512;  // four warpgroups: four threads per query row
constexpr int kTcEpiWarp0 = 20;         // warps 20-23: output epilogue
// Register budgets: launched at kTcLaunchRegs per thread; setmaxnreg moves
// registers from the producer/MMA warpgroup (kTcRegsIo) and the epilogue
// warpgroup (kTcRegsEpi) to the four softmax warpgroups (kTcRegsSoftmax).
// The split must fit in what the block was launched with (the host refuses
// to launch a build whose register count differs from kTcLaunchRegs).
constexpr int kTcLaunchRegs = 80, kTcRegsIo = 48, kTcRegsSoftmax = 96, kTcRegsEpi = 48;
static_assert(128 * kTcRegsIo + kTcSoftmaxThreads * kTcRegsSoftmax + 128 * kTcRegsEpi <= kTcThreads * kTcLaunchRegs,
              "register split");
constexpr int kTcMaxSlots = 10;

template <int D>
struct PrefillCfg {
  static constexpr int kAtoms = D / 64;                 // 128-byte column blocks per row
  static constexpr int kAtomBytes = kTcBlockM * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = kTcBlockM * D * 2;  // one 128-row tile of Q, K or V
  static constexpr int kSlots = D == 128 ? 5 : 10;
  static constexpr int kTilesBytes = (2 + kSlots) * kTileBytes;  // at the (1024-aligned) base
  static constexpr int kSmemBytes = kTilesBytes + 3072;           // + barriers and the row-max exchange
  static_assert(kSlots <= kTcMaxSlots, "slot count");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct PrefillCtrl {
  uint64_t q_full, q_empty;
  uint64_t slot_full[kTcMaxSlots], slot_empty[kTcMaxSlots];
  uint64_t s_full[2], p_full[2], o_done[2], o_empty[2];
  uint64_t l_ready, l_free;  // per unit: row sums handed to the epilogue warpgroup
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float xchg[4][kTcBlockM];  // (column group, row): partial row max / sum
};

// Wait-site codes reported in the workspace on a timeout.
enum : uint32_t {
  kSiteQEmpty = 0x101, kSiteSlotEmpty, kSiteQFull, kSiteSlotFull, kSitePFull, kSiteOEmpty,
  kSiteSFull, kSiteODone, kSiteDrain, kSiteLReady, kSiteLFree
};

struct UnitInfo {
  int b, m, h, g;
  SeqRange sr;
  int n[2];  // KV tiles needed by query tile 0 / 1
};

// The work of unit (b, m, h): its KV-tile counts per query tile.
__device__ __forceinline__ void unit_fill(const AttnParams &p, UnitInfo &ui) {
  ui.g = ui.h / (p.hq / p.hkv);
  ui.sr = seq_range(p, ui.b);
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first = ui.m * kTcUnitRows + t * kTcBlockM;
    if (first >= ui.sr.sq) {
      ui.n[t] = 0;
    } else {
      const int last = min(ui.sr.sq - 1, first + kTcBlockM - 1);
      ui.n[t] = (visible_keys(last, ui.sr.sq, ui.sr.sk, p.causal) + kTcBlockN - 1) / kTcBlockN;
    }
  }
}

// Unit u of the schedule.  Uniform lengths: 256-row blocks ordered by
// decreasing causal cost (last block first), all sequences of a block
// consecutively, heads innermost.  Varlen: the (b, m) pairs sorted by the
// prep kernel.
__device__ __forceinline__ UnitInfo unit_info(const AttnParams &p, int u) {
  UnitInfo ui;
  const int pr = u / p.hq;
  ui.h = u - pr * p.hq;
  if (p.cu_q == nullptr) {
    const int nblk = (p.sq + kTcUnitRows - 1) / kTcUnitRows;
    ui.m = nblk - 1 - pr / p.batch;
    ui.b = pr - (pr / p.batch) * p.batch;
  } else {
    const int2 pm = p.pairs[pr];
    ui.b = pm.x;
    ui.m = pm.y;
  }
  unit_fill(p, ui);
  return ui;
}

// Snake walk of the sorted unit list: round r, CTA c takes unit
// r*G + c (even r) or r*G + G-1-c (odd r).
__device__ __forceinline__ int unit_of(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

__device__ __forceinline__ int n_units_of(const AttnParams &p) {
  if (p.cu_q == nullptr) return p.batch * ((p.sq + kTcUnitRows - 1) / kTcUnitRows) * p.hq;
  return (int)(*reinterpret_cast<volatile uint32_t *>(&p.hdr->n_units)) * p.hq;
}

// The unit of this CTA's iteration `it` (false once the CTA has no more).
// Default: unit unit_of(it) of the list above (heaviest first, so the
// persistent CTAs finish close together).  Paired (p.paired, long causal
// sequences of uniform length with an even number of 256-row blocks): a work
// item is block nblk-1-k followed by block k of one (sequence, head), whose
// causal costs add up to the same number of KV tiles for every k; the items
// are dealt in the snake order with the k of one (sequence, head)
// consecutive, so the CTAs running at any time cover about 148 / (nblk/2)
// heads and their K/V streams share L2 instead of each head's K/V being
// re-read from DRAM by every block of it.
__device__ __forceinline__ bool unit_at(const AttnParams &p, int it, int cta, int grid, int n_units, UnitInfo &ui) {
  if (!p.paired) {
    const int u = unit_of(it, cta, grid);
    if (u >= n_units) return false;
    ui = unit_info(p, u);
    return true;
  }
  const int npairs = (p.sq + kTcUnitRows - 1) / kTcUnitRows / 2;
  const int item = unit_of(it >> 1, cta, grid);
  if (item >= n_units / 2) return false;
  const int bh = item / npairs, k = item - bh * npairs;
  ui.b = bh / p.hq;
  ui.h = bh - ui.b * p.hq;
  ui.m = (it & 1) ? k : 2 * npairs - 1 - k;
  unit_fill(p, ui);
  return true;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t pk2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Largest of N scores (-inf for none: masked keys are set to -inf before);
// four independent chains of three-input maxima.
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&sr)[N]) {
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int q = 0; q < N; q += 2)
    m4[(q >> 1) & 3] = fmax3(m4[(q >> 1) & 3], __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]));
  return fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
}

// P = 2^(c*s - base) for N scores, written into TMEM at taddr as packed
// 16-bit pairs (N/2 columns); returns the fp32 sum.  Score pairs go through
// the packed fp32x2 FMA; three of every eight pairs are exponentiated by the
// FMA-pipe polynomial, the rest by the multi-function unit.
template <bool MASKED, bool BF16, int N>
__device__ __forceinline__ float exp_store(const uint32_t (&sr)[N], int lim, float c, float base, uint32_t taddr) {
  const uint64_t c2 = pk2(__float_as_uint(c), __float_as_uint(c));
  const uint64_t nb2 = pk2(__float_as_uint(-base), __float_as_uint(-base));
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int q = 0; q < N / 32; ++q) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int c0 = q * 32 + 2 * e;
      const uint64_t x = ffma2(pk2(sr[c0], sr[c0 + 1]), c2, nb2);
      float p0, p1;
      if ((e & 7) >= 5) {
        upk2(exp2_poly2(x), p0, p1);
      } else {
        float x0, x1;
        upk2(x, x0, x1);
        p0 = ex2(x0);
        p1 = ex2(x1);
      }
      if (MASKED) {
        p0 = c0 < lim ? p0 : 0.f;
        p1 = c0 + 1 < lim ? p1 : 0.f;
      }
      acc[e & 3] = fadd2(acc[e & 3], pk2(__float_as_uint(p0), __float_as_uint(p1)));
      pk[e] = BF16 ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
    }
    tmem_st16(taddr + q * 16, pk);
  }
  tmem_wait_st();
  acc[0] = fadd2(acc[0], acc[1]);
  acc[2] = fadd2(acc[2], acc[3]);
  acc[0] = fadd2(acc[0], acc[2]);
  float lo, hi;
  upk2(acc[0], lo, hi);
  return lo + hi;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also returns the AND (bar_and) or OR (bar_or) of a
// per-thread predicate over the `count` participating threads.
__device__ __forceinline__ bool bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile("{\n .reg .pred q, p;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(r)
               : "r"((uint32_t)v), "r"(id), "r"(count)
               : "memory");
  return r != 0;
}
__device__ __forceinline__ bool bar_or(int id, int count, bool v) {
  uint32_t r;
  asm volatile("{\n .reg .pred q, p;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(r)
               : "r"((uint32_t)v), "r"(id), "r"(count)
               : "memory");
  return r != 0;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using Cfg = PrefillCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128B-swizzled tiles need a 1024-byte aligned base; the dynamic shared
  // memory of a kernel without static shared memory starts aligned.
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report_error(p.hdr, 2u /* MXFA_ERR_UNSUPPORTED */, 0x1FF);
    return;
  }
  PrefillCtrl *ctrl = reinterpret_cast<PrefillCtrl *>(smem_raw + Cfg::kTilesBytes);
  const uint32_t tiles_u32 = smem_u32(smem_raw);
  const uint32_t q_u32 = tiles_u32;                              // 2 query tiles
  const uint32_t ring_u32 = tiles_u32 + 2 * Cfg::kTileBytes;     // kSlots KV slots

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &ctrl->abort;
  WsHeader *hdr = p.hdr;

  const uint32_t b_qf = smem_u32(&ctrl->q_full), b_qe = smem_u32(&ctrl->q_empty);
  auto b_sf = [&](int s) { return smem_u32(&ctrl->slot_full[s]); };
  auto b_se = [&](int s) { return smem_u32(&ctrl->slot_empty[s]); };

  if (threadIdx.x == 0) {
    mbar_init(b_qf, 1);
    mbar_init(b_qe, 1);
    for (int s = 0; s < Cfg::kSlots; ++s) {
      mbar_init(b_sf(s), 1);
      mbar_init(b_se(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&ctrl->s_full[t]), 1);
      mbar_init(smem_u32(&ctrl->p_full[t]), kTcSoftmaxThreads / 32);  // one arrival per softmax warp
      mbar_init(smem_u32(&ctrl->o_done[t]), 1);
      mbar_init(smem_u32(&ctrl->o_empty[t]), 4);  // the epilogue warps
    }
    mbar_init(smem_u32(&ctrl->drain), 1);
    mbar_init(smem_u32(&ctrl->l_ready), 4);  // softmax warps of column group 0
    mbar_init(smem_u32(&ctrl->l_free), 4);   // the epilogue warps
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
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

  const int n_units = n_units_of(p);
  const int grid = gridDim.x, cta = blockIdx.x;

  if (warp < 4) {
  if constexpr (kTcRegsIo != kTcLaunchRegs) regs_dec<kTcRegsIo>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t ring = 0, q_issued = 0;
      bool ok = true;
      UnitInfo ui;
      for (int it = 0; ok && unit_at(p, it, cta, grid, n_units, ui); ++it) {
        const int nmax = max(ui.n[0], ui.n[1]);
        if (it > 0 && !wait_bar_flag(b_qe, (it - 1) & 1, abort_flag, kSiteQEmpty, p.wait_ns)) break;
        mbar_arrive_expect_tx(b_qf, 2 * Cfg::kTileBytes);
        const int qrow = ui.sr.q0 + ui.m * kTcUnitRows;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int a = 0; a < Cfg::kAtoms; ++a)
            tma_load_3d(q_u32 + t * Cfg::kTileBytes + a * Cfg::kAtomBytes, &tm_q, b_qf, a * 64, ui.h,
                        qrow + t * kTcBlockM);
        ++q_issued;
        for (int j = 0; j < nmax && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++ring) {
            const int s = ring % Cfg::kSlots;
            if (!wait_bar_flag(b_se(s), ((ring / Cfg::kSlots) & 1) ^ 1, abort_flag, kSiteSlotEmpty, p.wait_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(b_sf(s), Cfg::kTileBytes);
            const CUtensorMap *tm = kv ? &tm_v : &tm_k;
#pragma unroll
            for (int a = 0; a < Cfg::kAtoms; ++a)
              tma_load_3d(ring_u32 + s * Cfg::kTileBytes + a * Cfg::kAtomBytes, tm, b_sf(s), a * 64, ui.g,
                          ui.sr.k0 + j * kTcBlockN);
          }
        }
      }
      // Teardown: every load this thread issued must have landed before the
      // CTA exits (on the normal path they were all consumed already).
      const uint64_t t0 = global_ns();
      if (q_issued > 0)
        while (!mbar_test(b_qf, (q_issued - 1) & 1) && global_ns() - t0 < p.wait_ns) {
        }
      for (int s = 0; s < Cfg::kSlots; ++s) {
        const uint32_t uses = ring / Cfg::kSlots + ((uint32_t)s < ring % Cfg::kSlots ? 1u : 0u);
        if (uses == 0) continue;
        while (!mbar_test(b_sf(s), (uses - 1) & 1) && global_ns() - t0 < p.wait_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule, so MMA operands are computed
    // warp-uniformly; one elected lane issues each tcgen05 operation.
    const bool leader = elect_one();
    // every lane waits; the warp gives up together if any lane gave up
    auto wait_warp = [&](uint32_t bar, uint32_t parity, uint32_t site) {
      return __all_sync(0xffffffffu, wait_bar_flag(bar, parity, abort_flag, site, p.wait_ns));
    };
    {
      constexpr uint32_t idesc_s = make_idesc_f16(BF16, kTcBlockM, kTcBlockN, false, false);
      constexpr uint32_t idesc_o = make_idesc_f16(BF16, kTcBlockM, D, false, true);
      uint32_t ring = 0, p_cnt[2] = {0, 0}, o_uses[2] = {0, 0};
      // Descriptors: the high halves are fixed, a K-step only moves the
      // start address in the low half (16-byte units, never carries).
      const uint32_t sd_hi = desc_hi(make_sdesc_sw128(q_u32, 16, 1024));
      const uint32_t vd_hi = desc_hi(make_sdesc_sw128(ring_u32, Cfg::kAtomBytes, 1024));
      const uint32_t ring_lo = desc_lo(make_sdesc_sw128(ring_u32, 16, 1024));
      const uint32_t vring_lo = desc_lo(make_sdesc_sw128(ring_u32, Cfg::kAtomBytes, 1024));
      const uint32_t q_lo0 = desc_lo(make_sdesc_sw128(q_u32, 16, 1024));
      const uint32_t tm_base = __shfl_sync(0xffffffffu, tmem, 0);
      const uint32_t s_tm[2] = {tm_base, tm_base + kTcBlockN};
      const uint32_t o_tm[2] = {tm_base + 2 * kTcBlockN, tm_base + 2 * kTcBlockN + D};
      auto issue_s = [&](int t, int slot) {
        const uint32_t k_lo = ring_lo + (uint32_t)((slot * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          if (leader) mma_ss2(s_tm[t], q_lo0 + (uint32_t)((t * Cfg::kTileBytes + (kk >> 2) * Cfg::kAtomBytes + (kk & 3) * 32) >> 4), sd_hi,
                  k_lo + (uint32_t)((((kk >> 2) * Cfg::kAtomBytes) + (kk & 3) * 32) >> 4), sd_hi, idesc_s, kk > 0 ? 1u : 0u);
        if (leader) mma_commit(smem_u32(&ctrl->s_full[t]));
      };
      auto issue_pv = [&](int t, int slot, bool acc, bool last) {
        const uint32_t v_lo = vring_lo + (uint32_t)((slot * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTcBlockN / 16; ++kk)
          if (leader) mma_ts2(o_tm[t], s_tm[t] + (kk >> 1) * 32 + (kk & 1) * 8, v_lo + (uint32_t)(kk * 128), vd_hi, idesc_o,
                  (acc || kk > 0) ? 1u : 0u);
        if (leader && last) mma_commit(smem_u32(&ctrl->o_done[t]));  // O_t of the unit is complete
      };
      int it = 0;
      bool ok = true;
      UnitInfo ui;
      for (; ok && unit_at(p, it, cta, grid, n_units, ui); ++it) {
        const int nmax = max(ui.n[0], ui.n[1]);
        if (!wait_warp(b_qf, it & 1, kSiteQFull)) break;
        tc_fence_after();
        if (nmax == 0) {
          if (leader) mma_commit(b_qe);
          continue;
        }
        // prologue: S_t(0)
        {
          const int ks = ring % Cfg::kSlots;
          if (!wait_warp(b_sf(ks), (ring / Cfg::kSlots) & 1, kSiteSlotFull)) break;
          ++ring;
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (ui.n[t] > 0) issue_s(t, ks);
          if (leader) mma_commit(b_se(ks));
          if (nmax == 1 && leader) mma_commit(b_qe);
        }
        for (int j = 0; j < nmax && ok; ++j) {
          const int vs = ring % Cfg::kSlots;
          if (!wait_warp(b_sf(vs), (ring / Cfg::kSlots) & 1, kSiteSlotFull)) {
            ok = false;
            break;
          }
          ++ring;
          tc_fence_after();
          const bool has_next = j + 1 < nmax;
          int ks = -1;
          uint32_t kph = 0;
          bool kwaited = false;
          if (has_next) {
            ks = ring % Cfg::kSlots;
            kph = (ring / Cfg::kSlots) & 1;
            ++ring;
          }
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= ui.n[t]) continue;
            if (!wait_warp(smem_u32(&ctrl->p_full[t]), p_cnt[t] & 1, kSitePFull)) {
              ok = false;
              break;
            }
            ++p_cnt[t];
            if (j == 0 && o_uses[t] > 0 &&
                !wait_warp(smem_u32(&ctrl->o_empty[t]), (o_uses[t] - 1) & 1, kSiteOEmpty)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(t, vs, j > 0, j + 1 == ui.n[t]);
            if (j + 1 < ui.n[t]) {
              if (!kwaited) {
                if (!wait_warp(b_sf(ks), kph, kSiteSlotFull)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                kwaited = true;
              }
              issue_s(t, ks);
            }
          }
          if (!ok) break;
          if (leader) mma_commit(b_se(vs));
          if (has_next && leader) mma_commit(b_se(ks));
          if (j == nmax - 2 && leader) mma_commit(b_qe);
        }
        if (!ok) break;
        for (int t = 0; t < 2; ++t)
          if (ui.n[t] > 0) ++o_uses[t];
      }
      // Teardown: all MMAs issued by the elected lane complete before TMEM is freed.
      if (leader) mma_commit(smem_u32(&ctrl->drain));
      const uint64_t t0 = global_ns();
      while (!mbar_test(smem_u32(&ctrl->drain), 0) && global_ns() - t0 < p.wait_ns) {
      }
    }
  }
  } else if (warp < kTcEpiWarp0) {
    if constexpr (kTcRegsSoftmax != kTcLaunchRegs) regs_inc<kTcRegsSoftmax>();
    // ------------------------------------------------------------ softmax / epilogue
    // Four threads per query row, one per 32-key column group g; the four
    // warps of a TMEM sub-partition take both query tiles in turn, so every
    // score is read from TMEM once and stays in registers.
    const int g = (warp - 4) >> 2;  // column group: keys [32g, 32g+32), output columns [g*D/4, (g+1)*D/4)
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const int bar_id = 1 + sub;     // the four warps of this sub-partition
    constexpr int OC = D / 4;       // output columns per thread
    const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16);
    // A negative scale is handled by negating the scores in registers and
    // using |scale*log2 e| (c*s = |c|*(-s)), so the row maximum has one form.
    const bool neg = p.scale_log2 < 0.f;
    const float c = fabsf(p.scale_log2);
    float *x_mine = &ctrl->xchg[g][r];
    uint32_t s_cnt[2] = {0, 0};
    int it = 0;
    bool ok = true;
    UnitInfo ui;
    for (; ok && unit_at(p, it, cta, grid, n_units, ui); ++it) {
      const int nmax = max(ui.n[0], ui.n[1]);
      int i[2], nv[2];
      float m_used[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      {
        // the exchange area holds the previous unit's row sums until the
        // epilogue warpgroup has taken them
        bool lf = true;
        if (it > 0) lf = wait_bar_flag(smem_u32(&ctrl->l_free), (it - 1) & 1, abort_flag, kSiteLFree, p.wait_ns);
        __syncwarp();
        if (bar_or(bar_id, 128, !__all_sync(0xffffffffu, lf))) break;
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        i[t] = ui.m * kTcUnitRows + t * kTcBlockM + r;
        nv[t] = i[t] < ui.sr.sq ? visible_keys(i[t], ui.sr.sq, ui.sr.sk, p.causal) : 0;
      }
      for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (j >= ui.n[t]) continue;
          // A failed wait does not leave the loop here: the four warps of the
          // sub-partition first agree on it at the next named barrier, so
          // none is left waiting there for a warp that has gone.
          const bool got_s = wait_bar_flag(smem_u32(&ctrl->s_full[t]), s_cnt[t] & 1, abort_flag, kSiteSFull, p.wait_ns);
          __syncwarp();
          const bool wok = __all_sync(0xffffffffu, got_s);
          ++s_cnt[t];
          tc_fence_after();
          const uint32_t s_addr = trow + t * kTcBlockN + g * 32;
          const int lim = nv[t] - j * kTcBlockN - g * 32;  // keys [0, lim) of this group are visible
          const bool masked = __any_sync(0xffffffffu, lim < 32);
          uint32_t sa[32];
          tmem_ld32(s_addr, sa);
          if (neg) {
#pragma unroll
            for (int e = 0; e < 32; ++e) sa[e] ^= 0x80000000u;
          }
          if (masked) {  // keys >= lim to -inf (their P is set to 0 by exp_store as well)
#pragma unroll
            for (int e = 0; e < 32; ++e) sa[e] = e < lim ? sa[e] : 0xff800000u;
          }
          // this group's largest c*s.  One form of the reduction for all
          // tiles: with variants for masked tiles and negative scales the
          // softmax loop was longer and missed more in the instruction cache.
          const float ext = row_max<32>(sa);
          const float pm = (ext == -INFINITY) ? -INFINITY : ext * c;
          float alpha = 1.f;
          bool need = false;
          // Fast path: the stale base still bounds every group of every row
          // of this sub-partition (no row grew by more than 2^8).
          if (!bar_and(bar_id, 128, wok && m_used[t] != -INFINITY && pm <= m_used[t] + 8.f)) {
            if (bar_or(bar_id, 128, !wok)) {
              ok = false;
              break;
            }
            *x_mine = pm;
            named_bar_sync(bar_id, 128);
            const float mt = fmaxf(fmaxf(ctrl->xchg[0][r], ctrl->xchg[1][r]), fmaxf(ctrl->xchg[2][r], ctrl->xchg[3][r]));
            named_bar_sync(bar_id, 128);  // all have read before any writes again
            const float m_new = fmaxf(m_used[t], mt);
            if (m_used[t] == -INFINITY) {
              m_used[t] = m_new;  // nothing accumulated yet
            } else if (m_new > m_used[t] + 8.f) {
              alpha = ex2(m_used[t] - m_new);
              m_used[t] = m_new;
              need = true;
            }
          }
          const float base = (m_used[t] == -INFINITY) ? 0.f : m_used[t];
          // P = 2^(c*s - base) written as 16 packed columns at the start of
          // this group's own S columns
          const float rsum = masked ? exp_store<true, BF16, 32>(sa, lim, c, base, s_addr)
                                    : exp_store<false, BF16, 32>(sa, lim, c, base, s_addr);
          l[t] = l[t] * alpha + rsum;
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            // Rescale O_t.  PV_t(j-1), its latest accumulation, is complete:
            // it was issued before S_t(j), and the commit that signalled
            // S_t(j) tracks every earlier MMA of the issuing thread.
            // (rare: 16-column pieces in a rolled loop, for code size)
            const uint32_t oa = trow + 2 * kTcBlockN + t * D + g * OC;
#pragma unroll 1
            for (int h16 = 0; h16 < OC / 16; ++h16) {
              uint32_t ov[16];
              tmem_ld16(oa + h16 * 16, ov);
#pragma unroll
              for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
              tmem_st16(oa + h16 * 16, ov);
            }
            tmem_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&ctrl->p_full[t]));
        }
      }
      if (!ok) break;
      // Row sums over the four groups and the LSE; the sums go to the
      // epilogue warpgroup through the exchange area (xchg[t][row]).
      float lt[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        *x_mine = l[t];
        named_bar_sync(bar_id, 128);
        lt[t] = (ctrl->xchg[0][r] + ctrl->xchg[1][r]) + (ctrl->xchg[2][r] + ctrl->xchg[3][r]);
        named_bar_sync(bar_id, 128);  // all have read before the hand-over is written
        if (i[t] < ui.sr.sq && g == 0 && p.lse)
          p.lse[(int64_t)(ui.sr.q0 + i[t]) * p.hq + ui.h] =
              lt[t] > 0.f ? (m_used[t] + __log2f(lt[t])) * 0.69314718055994530942f : -INFINITY;
      }
      if (g == 0) {
        ctrl->xchg[0][r] = lt[0];
        ctrl->xchg[1][r] = lt[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctrl->l_ready));
      }
    }
  } else {
    if constexpr (kTcRegsEpi != kTcLaunchRegs) regs_dec<kTcRegsEpi>();
    // ------------------------------------------------------------ output epilogue
    // Warps 20-23, one thread per query row (warp w reads TMEM lanes
    // 32*(w%4)..+31): O_t / l in the output dtype once the unit's last P.V of
    // tile t is complete; then O_t's TMEM columns are released to the MMAs.
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16);
    const bool o_v8 = ((reinterpret_cast<uintptr_t>(p.o) | (uintptr_t)(p.o_rs * 2) | (uintptr_t)(p.o_hs * 2)) & 31u) == 0;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    uint32_t o_cnt[2] = {0, 0};
    bool ok = true;
    UnitInfo ui;
    for (int it = 0; ok && unit_at(p, it, cta, grid, n_units, ui); ++it) {
      const bool got_l = wait_bar_flag(smem_u32(&ctrl->l_ready), it & 1, abort_flag, kSiteLReady, p.wait_ns);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got_l)) break;
      const float lt0 = ctrl->xchg[0][r], lt1 = ctrl->xchg[1][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctrl->l_free));
      // Rolled loops (the tile state selected, not indexed): this warpgroup
      // shares the SM sub-partitions with the softmax warps, and its code,
      // run once per unit, is kept small so the softmax loop stays in the
      // instruction cache (unrolled over both tiles and all column chunks it
      // cost 1.5-2 % on the 2K and varlen workloads).
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        const float lt = t ? lt1 : lt0;
        const int i = ui.m * kTcUnitRows + t * kTcBlockM + r;
        const bool valid = i < ui.sr.sq;
        T *orow = reinterpret_cast<T *>(p.o) + (int64_t)(ui.sr.q0 + i) * p.o_rs + (int64_t)ui.h * p.o_hs;
        if ((t ? ui.n[1] : ui.n[0]) > 0) {
          const uint32_t oc = t ? o_cnt[1] : o_cnt[0];
          const bool got_o = wait_bar_flag(smem_u32(&ctrl->o_done[t]), oc & 1, abort_flag, kSiteODone, p.wait_ns);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got_o)) {
            ok = false;
            break;
          }
          if (t) o_cnt[1] = oc + 1; else o_cnt[0] = oc + 1;
          tc_fence_after();
          const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t ov[16], pk[8];
            tmem_ld16(trow + 2 * kTcBlockN + t * D + c * 16, ov);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a0 = __uint_as_float(ov[2 * e]) * inv, a1 = __uint_as_float(ov[2 * e + 1]) * inv;
              pk[e] = BF16 ? pack_bf16x2(a0, a1) : pack_f16x2(a0, a1);
            }
            if (valid) {
              if (o_v8) {
                st_global_v8(orow + c * 16, pk);
              } else {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&ctrl->o_empty[t]));
        } else if (valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
          for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0, 0, 0, 0);
        }
      }
    }
  }

  __syncwarp();  // the single-lane roles rejoin their warps before the CTA barrier
  __syncthreads();
  // a wait that gave up left its site in the abort flag
  if (threadIdx.x == 0 && ctrl->abort) report_error(hdr, kStatusTimeout, (uint32_t)ctrl->abort);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mxfa
