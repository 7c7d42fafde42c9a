// decode_tc.cuh -- split-KV MLA decode on the tensor cores (sm_100a).
//
// Shape (kernelbot-amd-mixed-mla submission 588924, _flash_fused /
// _flash_splitk / _reduce_splitk): every sequence b has q_len queries of Hq
// heads that all read one shared latent KV row of 576 columns; the value is
// the first 512 columns of that same row.  The query heads are taken in head
// groups of G heads with q_len*G <= 64 (one group, G = Hq, when q_len*Hq <=
// 64); the q_len*G query rows of a group are flattened r = q*G + j (token q,
// head gh*G + j) and form the M = 64 side of every MMA.
//
// The KV cache is streamed exactly once: 64-key tiles arrive by TMA as nine
// 8 KB column chunks (64 keys x 64 columns, 128B swizzle) into a 27-slot
// ring (three tiles, so two tiles are in flight while one is computed).
// Each tile is used twice while resident:
//     S   = Q K^T   tcgen05.mma M=64 N=64, 36 K-steps, A = Q (TMEM), B = K;
//                   the K-steps go round-robin into three accumulators
//                   (chunk c into chain c % 3) so consecutive MMAs do not
//                   wait on each other; softmax adds the three
//     O  += P V     tcgen05.mma M=64 N=256 (x2), A = P (smem), B = chunks 0-7
// TMEM: O in lanes 0-15 of each sub-partition (all 512 columns); in lanes
// 16-31 the three S chains (columns 0-191) and Q (columns 192-479, two bf16
// per column), so the shared-memory budget goes to the KV ring.  S has one
// buffer: softmax signals as soon as it has read S(j), and S(j+1) is issued
// before P.V(j).  A softmax warpgroup (128 threads) gives each query row two threads,
// one per 32-key half of the tile (16-lane TMEM accesses), with the online
// softmax of the prefill kernel (exp2 domain, rescale of O only when the
// row max grows by more than 2^8).
//
// Work split (d1): the KV tiles of all sequences form one sequence of T
// tiles; CTA c of G owns the pieces whose first tile lies in
// [c*T/G, (c+1)*T/G).  Pieces are whole sequences, or (when that would
// leave the CTAs badly unbalanced) the sequences cut at those boundaries, or
// with num_splits = k every sequence cut into k near-equal pieces.  A sequence covered by
// one piece is normalised and stored directly; otherwise every piece writes
// its unnormalised partial (acc, running max, running sum) and
// decode_combine_kernel merges them with weights 2^(m_s - max_s m_s).
#pragma once

#include <type_traits>

#include <cub/block/block_scan.cuh>

#include "ptx.cuh"

namespace mxfa {

constexpr int kDcRows = 64;       // M: query rows per sequence
constexpr int kDcKeys = 64;       // keys per tile
constexpr int kDcDqk = 576, kDcDv = 512;
constexpr int kDcChunks = kDcDqk / 64;  // 9 column chunks per KV tile
constexpr int kDcChunkBytes = kDcKeys * 128;
constexpr int kDcRingTiles = 3;
constexpr int kDcSlots = kDcRingTiles * kDcChunks;
constexpr int kDcQCol = 192;  // first TMEM column of Q (lanes 16-31); S chains use 0-191
constexpr int kDcThreads = 256;
constexpr int kDcCtrlBytes = 2048;
constexpr int kDcSmemBytes = kDcCtrlBytes + kDcSlots * kDcChunkBytes + kDcRows * 128;
static_assert(kDcSmemBytes <= 232448, "shared memory budget");
constexpr int kDcMaxGrid = 256;
// The decode kernels have no register split: their error reports are calls.
constexpr bool kDcColdReport = true;

// A decode "sequence" v is (batch entry b, head group gh) (dc_seq): the
// G = Hq/heads query heads gh*G .. gh*G+G-1 of b, which read KV head
// gh / subs.  heads = Hkv * subs: 1 for MLA (all query heads share the one
// latent KV head), Hkv for grouped-query decode (the query heads of KV head
// g); subs > 1 splits each KV head's query heads into subs groups when
// q_len * Hq/Hkv exceeds the 64 query rows of the MMAs.  Each group streams
// the KV head again; the sequences are numbered group-major (all batch
// entries of group 0, then of group 1, ...), so the groups of one batch
// entry land on CTAs far apart in the tile order and read the same tiles at
// about the same time, the later reads from L2.
// n / d for 0 <= n < 2^31 as (n * m) >> sh with sh = 31 + ceil(log2 d) and
// m = ceil(2^sh / d) (the round-up method of division by invariant integers,
// Granlund and Montgomery 1994): exact because n * (m * d - 2^sh) < 2^31 * d
// <= 2^sh.  A multiply and a shift in place of a division sequence.
struct DivU {
  uint32_t m, sh;
  int d;
};
__device__ __forceinline__ int div_u(int n, const DivU &q) { return (int)(((uint64_t)(uint32_t)n * q.m) >> q.sh); }

struct DecodeSched {
  int heads;       // head groups per batch entry that form separate sequences
  int subs;        // head groups per KV head
  int keys;        // keys per KV tile
  int *n_tiles;    // [batch*heads] KV tiles per sequence
  int *tile_pre;   // [batch*heads + 1] prefix of n_tiles
  int *seg_base;   // [batch*heads + 1] first segment of each sequence
  int *seg_cnt;    // [batch*heads]
  int4 *segs;      // [max_segs] (v, first tile, end tile, global first tile)
  float *part_acc; // [max_segs][64][Dv]
  float2 *part_ml; // [max_segs][64] (running max in log2 units, running sum)
  int max_segs;
  int num_splits;  // 0 = automatic
  // Automatic schedule: whole sequences are kept while the longest CTA of
  // that deal is within whole_pct % of the even cut (a split piece costs a
  // partial of 64 rows x Dv fp32 written and re-read, and a combine pass).
  int whole_pct;
  int grid;
  // KV-cache mode (p.cu_k == nullptr): batch entry b has cache_seqlens[b] + add
  // keys; key position pos is cache row b*page_size + pos (dense cache,
  // block_table == nullptr) or block_table[b][pos / page_size]*page_size +
  // pos % page_size (paged).  The prep kernel writes the key counts to
  // kv_len and, when advance != 0, then adds `add` to cache_seqlens.
  int32_t *cache_seqlens;
  int add, advance;
  int *kv_len;
  const int32_t *block_table;
  int max_blocks, page_size;
  // Single-launch schedule (arith_k > 0, packed kv_indptr only): sequence v
  // is cut into k_v = min(arith_k, its KV tiles) near-equal pieces and piece
  // i is CTA v*arith_k + i, so no prep kernel runs.  The pieces of a split
  // sequence merge their partials at the end of the same kernel; sync[v]
  // counts the pieces that have stored theirs (zeroed before the launch).
  int arith_k;
  int *sync;
  // Schedule kernel output: the number of sequences not stored directly by
  // the decode kernel (split into pieces, or with no piece at all); the
  // combine kernel has nothing to do when it is 0.
  int *n_multi;
  // Factor of every stored output and partial accumulator: 1, or the KV
  // dequantisation scale of the fp8-KV MLA kernel (the scores' share of that
  // scale is folded into AttnParams::scale_log2 by the host).
  float o_scale;
  DivU by_bh, by_hkv;  // divisors of dc_seq: batch * Hkv and Hkv
};

struct DcSeq {
  int b, gh, kvh;  // batch entry, head group, KV head
};
// v = (sub * batch + b) * Hkv + kvh with gh = kvh * subs + sub.
__device__ __forceinline__ DcSeq dc_seq(const AttnParams &p, const DecodeSched &s, int v) {
  const int sub = div_u(v, s.by_bh), w = v - sub * s.by_bh.d;
  DcSeq r;
  r.b = div_u(w, s.by_hkv);
  r.kvh = w - r.b * s.by_hkv.d;
  r.gh = r.kvh * s.subs + sub;
  return r;
}

// Queries of batch entry b: (first row, count); packed (cu_q) or uniform.
__device__ __forceinline__ int2 dc_q(const AttnParams &p, int b) {
  if (p.cu_q) return make_int2(p.cu_q[b], p.cu_q[b + 1] - p.cu_q[b]);
  return make_int2(b * p.max_sq, p.max_sq);
}
// Keys of batch entry b.
__device__ __forceinline__ int dc_klen(const AttnParams &p, const DecodeSched &s, int b) {
  return p.cu_k ? p.cu_k[b + 1] - p.cu_k[b] : s.kv_len[b];
}
// Cache row of key position pos (< its key count) of batch entry b, or an
// out-of-range row (read as zeros by TMA) when the block table has no page
// for it.
__device__ __forceinline__ int dc_krow(const AttnParams &p, const DecodeSched &s, int b, int pos) {
  if (p.cu_k) return p.cu_k[b] + pos;
  if (!s.block_table) return b * s.page_size + pos;
  const int idx = pos / s.page_size;
  if (idx >= s.max_blocks) return -(1 << 30);
  const int page = s.block_table[(int64_t)b * s.max_blocks + idx];
  return page < 0 ? -(1 << 30) : page * s.page_size + pos % s.page_size;
}

struct DecodeCtrl {
  uint64_t q_ready;
  uint64_t tile_full[kDcRingTiles], tile_empty[kDcRingTiles];
  uint64_t stage_full[kDcRingTiles];  // fp8 KV: the codes of chunks 0-2 of the slot have landed
  uint64_t stage_rest[kDcRingTiles];  // fp8 KV: the codes of chunks 3-8 have landed
  uint64_t low_full[kDcRingTiles];    // fp8 KV: bf16 chunks 0-2 of the slot are written
  uint64_t s_full, s_free, p_full, o_done, o_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

enum : uint32_t {
  kDSiteSlotEmpty = 0x301, kDSiteQReady, kDSiteSlotFull, kDSitePFull, kDSiteOEmpty, kDSiteSFull,
  kDSiteODone, kDSiteSFree, kDSiteMerge, kDSiteStageFull
};

__device__ __forceinline__ int dc_range_start(int c, int T, int G) { return (int)(((int64_t)c * T) / G); }

// Programmatic dependent launch.  The decode kernel (after the schedule
// kernel) and the combine kernel (after the decode kernel) are launched with
// programmatic stream serialisation, so their CTAs may become resident while
// the kernel before them still runs: dc_pdl_wait() blocks until that kernel
// has completed and its writes are visible, and dc_pdl_release() lets the
// next kernel's CTAs launch.  Without such a dependency both are no-ops.
__device__ __forceinline__ void dc_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void dc_pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Four outputs, rounded to the 16-bit output type, as one 8-byte store.
template <typename T>
__device__ __forceinline__ void dc_store4(T *dst, float a, float b, float c, float d) {
  uint32_t lo, hi;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    lo = pack_bf16x2(a, b);
    hi = pack_bf16x2(c, d);
  } else {
    lo = pack_f16x2(a, b);
    hi = pack_f16x2(c, d);
  }
  *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
}

// Partial accumulator of piece sg, row r, columns 4*c4 .. 4*c4+3: layout
// [piece][DV/4][64 rows] in float4 units, so the threads that hold
// consecutive rows of the same four columns touch consecutive 16-byte words.
template <int DV>
__device__ __forceinline__ float4 *dc_pacc(const DecodeSched &s, int sg, int r, int c4) {
  return reinterpret_cast<float4 *>(s.part_acc) + ((int64_t)sg * (DV / 4) + c4) * kDcRows + r;
}

// KV tiles of decode sequence v (0 when its batch entry has no query).
__device__ __forceinline__ int dc_seq_tiles(const AttnParams &p, const DecodeSched &s, int v) {
  const int b = dc_seq(p, s, v).b;
  if (dc_q(p, b).y <= 0) return 0;
  return (dc_klen(p, s, b) + s.keys - 1) / s.keys;
}
// Pieces of sequence v.
__device__ __forceinline__ int dc_seg_cnt(const AttnParams &p, const DecodeSched &s, int v) {
  return s.arith_k > 0 ? min(s.arith_k, dc_seq_tiles(p, s, v)) : s.seg_cnt[v];
}
// Piece sg: (sequence, first tile, end tile, global first tile; the last
// is not used by the single-launch schedule).
__device__ __forceinline__ int4 dc_seg(const AttnParams &p, const DecodeSched &s, int sg) {
  if (s.arith_k == 0) return s.segs[sg];
  const int v = sg / s.arith_k, i = sg % s.arith_k;
  const int n = dc_seq_tiles(p, s, v), k = max(1, min(s.arith_k, n));
  return make_int4(v, (int)(((int64_t)i * n) / k), (int)(((int64_t)(i + 1) * n) / k), 0);
}

// First segment whose first global tile is >= x.
__device__ __forceinline__ int dc_lower_bound(const int4 *segs, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (segs[mid].w < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// ----------------------------------------------------------------------------
// Schedule: one 1024-thread CTA.
//   n_tiles[b]   = ceil(kv_len_b / keys) (0 when the sequence has no queries)
//   tile_pre     = prefix of n_tiles (the global tile sequence)
//   pieces       = num_splits > 0: min(k, n_b) near-equal pieces per sequence;
//                  automatic: whole sequences, unless cutting the global tile
//                  sequence at the CTA boundaries c*T/G shortens the longest
//                  CTA by more than DecodeSched::whole_pct allows (splitting
//                  costs partial writes, a combine pass and an extra Q load
//                  per piece).
__global__ void __launch_bounds__(1024) decode_prep_kernel(const AttnParams p, DecodeSched s) {
  dc_pdl_release();  // the decode kernel's CTAs may set up while this runs
  using Scan = cub::BlockScan<int, 1024>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int carry, max_n, split_mode, n_multi;
  __shared__ int cut[kDcMaxGrid + 1];  // x_c = c*T/G, c = 0..G
  __shared__ int ps[kDcMaxGrid + 1];   // ps[c]: c' in [1, c] with cut[c'] != cut[c'-1] (distinct cut values)
  const int tid = threadIdx.x, B = p.batch * s.heads, G = s.grid;
  if (tid == 0) {
    carry = 0;
    max_n = 0;
    n_multi = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int b = base + tid;
    int n = 0;
    if (b < B) {
      const DcSeq sq_b = dc_seq(p, s, b);
      const int e = sq_b.b;  // batch entry of sequence b
      int len = p.cu_k ? p.cu_k[e + 1] - p.cu_k[e] : s.cache_seqlens[e] + s.add;
      if (!p.cu_k) {
        // A cache entry holds at most page_size keys (dense) or max_blocks
        // pages (paged); positions beyond would read another entry's rows or
        // no page at all, so the length is cut there and the call reports it.
        const int64_t cap = s.block_table ? (int64_t)s.max_blocks * s.page_size : (int64_t)s.page_size;
        if (len > cap) {
          if (sq_b.gh == 0) report_error_cold(p.hdr, 1u /* MXFA_ERR_INVALID_ARG */, 0x402);
          len = (int)cap;
        }
        if (sq_b.gh == 0) s.kv_len[e] = len;
      }
      n = (len + s.keys - 1) / s.keys;
      if (dc_q(p, e).y <= 0) n = 0;  // no queries: nothing to compute
      s.n_tiles[b] = n;
    }
    // one shared atomic per warp (all lanes reach here; n = 0 past B)
    const int wmax = __reduce_max_sync(0xffffffffu, n);
    if ((tid & 31) == 0 && wmax > 0) atomicMax(&max_n, wmax);
    int incl, total;
    Scan(tmp).InclusiveSum(n, incl, total);
    if (b < B) s.tile_pre[b + 1] = carry + incl;
    __syncthreads();
    if (tid == 0) carry += total;
    __syncthreads();
  }
  if (tid == 0) s.tile_pre[0] = 0;
  const int T = carry;
  if (!p.cu_k && s.advance)  // every read of cache_seqlens above is done
    for (int e = tid; e < p.batch; e += 1024) s.cache_seqlens[e] += s.add;
  for (int c = tid; c <= G; c += 1024) cut[c] = (int)(((int64_t)c * T) / G);
  if (tid == 0) {
    // longest CTA with whole sequences (they are dealt out by first tile) vs. the even cut
    const int64_t whole = (int64_t)max_n * ((B + G - 1) / G);
    const int64_t even = (T + G - 1) / G;
    split_mode = (s.num_splits > 0) ? 1 : (100 * whole > s.whole_pct * even ? 2 : 0);  // 0 whole, 1 k pieces, 2 even cut
  }
  __syncthreads();
  {
    int incl, total;
    Scan(tmp).InclusiveSum((tid >= 1 && tid <= G && cut[tid] != cut[tid - 1]) ? 1 : 0, incl, total);
    if (tid <= G) ps[tid] = incl;
  }
  __syncthreads();
  // first c with cut[c] > x / with cut[c] >= x (cut is non-decreasing)
  auto upper = [&](int x) {
    int lo = 0, hi = G + 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (cut[mid] <= x) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  auto lower = [&](int x) {
    int lo = 0, hi = G + 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (cut[mid] < x) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  auto pieces = [&](int b) -> int {
    const int n = s.n_tiles[b];
    if (n == 0) return 0;
    if (split_mode == 0) return 1;
    if (split_mode == 1) return min(s.num_splits, n);
    // 1 + the distinct cut values strictly inside (P, P + n); the first cut
    // above P always differs from the one before it
    const int P = s.tile_pre[b];
    const int lo = upper(P), hi = lower(P + n);
    return 1 + (hi > lo ? ps[hi - 1] - ps[lo - 1] : 0);
  };
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int b = base + tid;
    const int k = b < B ? pieces(b) : 0;
    if (b < B) s.seg_cnt[b] = k;
    const int wmulti = (int)__reduce_add_sync(0xffffffffu, (b < B && k != 1) ? 1u : 0u);
    if ((tid & 31) == 0 && wmulti > 0) atomicAdd(&n_multi, wmulti);
    int incl, total;
    Scan(tmp).InclusiveSum(k, incl, total);
    if (b < B) s.seg_base[b] = carry + incl - k;
    __syncthreads();
    if (tid == 0) carry += total;
    __syncthreads();
  }
  const int n_segs = carry;
  if (tid == 0) s.seg_base[B] = n_segs;
  __syncthreads();
  // Segment list.  Each sequence writes its first piece (and, in modes 0
  // and 1, all of them); in mode 2 every distinct cut value strictly inside
  // a sequence writes the piece it starts, so no thread walks a long run of
  // cuts.
  for (int b = tid; b < B; b += 1024) {
    const int n = s.n_tiles[b], P = s.tile_pre[b], k = s.seg_cnt[b];
    const int idx = s.seg_base[b];
    if (k == 0) continue;
    if (split_mode == 1) {
      for (int i = 0; i < k; ++i) {
        const int t0 = (int)(((int64_t)i * n) / k), t1 = (int)(((int64_t)(i + 1) * n) / k);
        if (idx + i < s.max_segs) s.segs[idx + i] = make_int4(b, t0, t1, P + t0);
      }
    } else {
      const int e0 = split_mode == 2 ? min(cut[upper(P)], P + n) : P + n;  // cut[G] = T > P
      if (idx < s.max_segs) s.segs[idx] = make_int4(b, 0, e0 - P, P);
    }
  }
  if (split_mode == 2) {
    for (int c = 1 + tid; c < G; c += 1024) {
      const int x = cut[c];
      if (x == cut[c - 1] || x <= 0 || x >= T) continue;
      // the sequence b with tile_pre[b] < x <= tile_pre[b + 1]
      int lo = 1, hi = B;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s.tile_pre[mid] < x) lo = mid + 1; else hi = mid;
      }
      const int b = lo - 1, P = s.tile_pre[b], n = s.n_tiles[b];
      if (x >= P + n) continue;  // x starts the next sequence: not a cut inside b
      const int k = ps[c] - ps[upper(P) - 1];  // this piece's index within b (>= 1)
      const int e = min(cut[upper(x)], P + n);
      const int idx = s.seg_base[b] + k;
      if (idx < s.max_segs) s.segs[idx] = make_int4(b, x - P, e - P, x);
    }
  }
  __syncthreads();
  if (tid == 0) {
    p.hdr->n_units = (uint32_t)min(n_segs, s.max_segs);
    p.hdr->n_aux = (uint32_t)T;
    *s.n_multi = n_multi;
    if (n_segs > s.max_segs) report_error_cold(p.hdr, 1u /* MXFA_ERR_INVALID_ARG */, 0x401);
  }
}

// ----------------------------------------------------------------------------
// Single-launch schedule: merge of a split sequence at the end of the decode
// kernel.  Piece i of the k pieces of sequence v, once its partial is
// stored, announces it on s.sync[v] and waits (bounded) until all k have;
// it then merges slice i of the sequence's (row, 4-column) outputs with the
// weights 2^(m_t - M) of decode_combine_kernel.  The pieces of a sequence
// run at the same time (the kernel is launched cooperatively, one CTA per
// piece).  Every thread of the CTA calls it; `scratch` is shared memory no
// longer in use, 160 + 128 k floats.
template <typename T, int DV, int NT>
__device__ void dc_merge_pieces(const AttnParams &p, const DecodeSched &s, int v, int i, int k, float *scratch) {
  volatile int *flag = reinterpret_cast<volatile int *>(scratch);
  const DcSeq sq = dc_seq(p, s, v);
  const int b = sq.b, gh = sq.gh, G = p.hq / s.heads;
  const int2 qr = dc_q(p, b);
  const int rows = qr.y * G;
  // scratch: flag, then per row M and L, then the weights w and sums l of
  // every (row, piece)
  float *Mr = scratch + 32, *Lr = Mr + kDcRows, *w = Lr + kDcRows, *wl = w + rows * k;
  __threadfence();  // this thread's partial stores are visible to the other pieces
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(s.sync + v, 1);
    const uint64_t t0 = global_ns();
    int good = 1;
    while (*reinterpret_cast<volatile int *>(s.sync + v) < k) {
      if (global_ns() - t0 > p.wait_ns) {
        report_error_cold(p.hdr, kStatusTimeout, kDSiteMerge);
        good = 0;
        break;
      }
    }
    *flag = good;
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  constexpr int C4 = DV / 4;
  // This piece's slice of the (4-column group, row) items, rows fastest.
  const int n_items = rows * C4;
  const int lo = (int)(((int64_t)i * n_items) / k), hi = (int)(((int64_t)(i + 1) * n_items) / k);
  if (lo >= hi) return;
  const int base = v * s.arith_k;  // partial slot of piece 0
  // (m, l) of every (piece t, row r) at [t * rows + r], in one parallel
  // pass; then one thread per row turns the maxima into the weights
  // w = 2^(m - M) (in place) and the sum L.
  for (int e = threadIdx.x; e < rows * k; e += NT) {
    const float2 ml = s.part_ml[(int64_t)(base + e / rows) * kDcRows + e % rows];
    w[e] = ml.x;
    wl[e] = ml.y;
  }
  __syncthreads();
  for (int r = threadIdx.x; r < rows; r += NT) {
    float m = -INFINITY;
    for (int t = 0; t < k; ++t) m = fmaxf(m, w[t * rows + r]);
    float ls = 0.f;
    for (int t = 0; t < k; ++t) {
      const float wt = m == -INFINITY ? 0.f : ex2(w[t * rows + r] - m);  // 0 for a piece that saw no visible key
      w[t * rows + r] = wt;
      ls += wt * wl[t * rows + r];
    }
    Mr[r] = m;
    Lr[r] = ls;
  }
  __syncthreads();
  // This thread's items lo + threadIdx.x + q*NT, two at a time; the partial
  // loads of up to eight pieces of both are issued before any is used, so
  // up to sixteen are in flight.
  const int nq = hi - lo > (int)threadIdx.x ? (hi - lo - 1 - (int)threadIdx.x) / NT + 1 : 0;
  for (int q0 = 0; q0 < nq; q0 += 2) {
    const bool two = q0 + 1 < nq;
    int rq[2], cq[2];
    float4 acc[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int it = lo + threadIdx.x + (q0 + (two ? q : 0)) * NT;
      rq[q] = it % rows;
      cq[q] = it / rows;
      acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int t0 = 0; t0 < k; t0 += 8) {
      float4 a[2][8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int q = 0; q < 2; ++q)
          a[q][u] = t0 + u < k ? *dc_pacc<DV>(s, base + t0 + u, rq[q], cq[q]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float wt = t0 + u < k ? w[(t0 + u) * rows + rq[q]] : 0.f;
          acc[q].x = fmaf(wt, a[q][u].x, acc[q].x);
          acc[q].y = fmaf(wt, a[q][u].y, acc[q].y);
          acc[q].z = fmaf(wt, a[q][u].z, acc[q].z);
          acc[q].w = fmaf(wt, a[q][u].w, acc[q].w);
        }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (q == 1 && !two) break;
      const int r = rq[q], c4 = cq[q];
      const float L = Lr[r], inv = L > 0.f ? 1.f / L : 0.f;
      const int tok = qr.x + r / G, h = gh * G + r % G;
      T *orow = reinterpret_cast<T *>(p.o) + (int64_t)tok * p.o_rs + (int64_t)h * p.o_hs + 4 * c4;
      dc_store4<T>(orow, acc[q].x * inv, acc[q].y * inv, acc[q].z * inv, acc[q].w * inv);
      if (c4 == 0 && p.lse)
        p.lse[(int64_t)tok * p.hq + h] = L > 0.f ? (Mr[r] + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
  }
}

// Single-launch schedule: a sequence with no piece (no key, or no query)
// gets O = 0 and LSE = -inf, written by its CTA 0.
template <typename T, int DV, int NT>
__device__ void dc_zero_rows(const AttnParams &p, const DecodeSched &s, int v) {
  const DcSeq sq = dc_seq(p, s, v);
  const int b = sq.b, gh = sq.gh, G = p.hq / s.heads;
  const int2 qr = dc_q(p, b);
  const int rows = qr.y * G;
  for (int it = threadIdx.x; it < rows * DV; it += NT) {
    const int r = it / DV, c = it % DV;
    const int tok = qr.x + r / G, h = gh * G + r % G;
    reinterpret_cast<T *>(p.o)[(int64_t)tok * p.o_rs + (int64_t)h * p.o_hs + c] = from_f32<T>(0.f);
    if (c == 0 && p.lse) p.lse[(int64_t)tok * p.hq + h] = -INFINITY;
  }
}

// ----------------------------------------------------------------------------
// ----------------------------------------------------------------------------
// fp8 KV (OCP 8-bit floating point, E4M3: sign, 4 exponent bits with bias 7,
// 3 mantissa bits, subnormals, no infinities).  A tile's codes (nine
// unswizzled 64 keys x 64-byte column chunks, 36,864 bytes) land by TMA in
// the upper half of the ring slot that will hold the tile in bf16; six
// widening warps turn them in place into the nine 64 x 128-byte,
// 128B-swizzled bf16 chunks the MMA reads.  The bf16 chunks 0-3 end below
// the codes; chunks 4-8 overwrite codes, so every code is read into
// registers before any of those is written.
constexpr int kDcStageChunkBytes = kDcKeys * 64;
constexpr int kDcStageBytes = kDcChunks * kDcStageChunkBytes;  // 36,864
constexpr int kDcStageOff = kDcChunks * kDcChunkBytes - kDcStageBytes;  // codes: upper half of the slot
static_assert(4 * kDcChunkBytes <= kDcStageOff, "bf16 chunks 0-3 end below the staged codes");
constexpr int kDcThreadsFp8 = 384;  // + warps 8-11, which widen together with warps 2-3
constexpr int kDcWiden = 192;       // widening threads: warps 8-11, then 2-3
constexpr int kDcWidenLow = 3;      // bf16 chunks 0-2 are signalled before chunks 3-8
static_assert((kDcChunks * kDcKeys * 4) % kDcWiden == 0 && (kDcWidenLow * kDcKeys * 4) % kDcWiden == 0,
              "widening groups divide evenly");

// Four E4M3 codes (the bytes of w, lowest first) to four bf16 values, exactly.
// Code byte c becomes the 16-bit pattern sign(c) << 15 | (c & 0x7f) << 4: the
// E4M3 exponent and mantissa fields become the low four bits of bf16's
// exponent and the top three of its mantissa, i.e. the bf16 value is the E4M3
// value times 2^-120 (E4M3 subnormals become bf16 subnormals), and one bf16x2
// multiply by 2^120 restores it.  prmt builds (c, sign-fill(c)) byte pairs,
// so the shift puts the sign in bit 15; the mask clears the rest.  The two
// NaN codes (0x7f, 0xff) come out as +-480.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
  uint32_t a, b;
  asm("prmt.b32 %0, %1, 0, 0x9180;" : "=r"(a) : "r"(w));
  asm("prmt.b32 %0, %1, 0, 0xB3A2;" : "=r"(b) : "r"(w));
  a = (a << 4) & 0x87F087F0u;
  b = (b << 4) & 0x87F087F0u;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0x7B807B80u));  // 0x7B80 = 2^120
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0x7B807B80u));
}

// FP8 = true: the KV cache holds E4M3 codes (tm_kv is a byte map, box 64 x 64,
// no swizzle), staged in the ring slots and widened there by warps 8-11 and
// 2-3 (384 threads); from there the MMA and softmax roles run unchanged.  The
// dequantisation scale multiplies the scores (through p.scale_log2) and the
// outputs (s.o_scale).
template <bool BF16, bool FP8 = false>
__global__ void __launch_bounds__(FP8 ? kDcThreadsFp8 : kDcThreads, 1)
attn_decode_tc_kernel(const __grid_constant__ AttnParams p, const DecodeSched s,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv) {
  static_assert(!FP8 || BF16, "fp8 KV is widened to bf16");
  constexpr int RT = kDcRingTiles;
  extern __shared__ uint8_t smem_raw[];
  DecodeCtrl *ctrl = reinterpret_cast<DecodeCtrl *>(smem_raw);
  const uint32_t tiles_u32 = (smem_u32(smem_raw) + 1024u + 1023u) & ~1023u;
  const uint32_t ring_u32 = tiles_u32;                               // RT tiles x 9 KV chunks
  const uint32_t p_u32 = ring_u32 + kDcSlots * kDcChunkBytes;        // P: 64 rows x 128 B
  uint8_t *p_gen = smem_raw + (p_u32 - smem_u32(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &ctrl->abort;
  WsHeader *hdr = p.hdr;
  auto b_tf = [&](int x) { return smem_u32(&ctrl->tile_full[x]); };
  auto b_te = [&](int x) { return smem_u32(&ctrl->tile_empty[x]); };
  auto b_gf = [&](int x) { return smem_u32(&ctrl->stage_full[x]); };
  auto b_gr = [&](int x) { return smem_u32(&ctrl->stage_rest[x]); };
  auto b_lf = [&](int x) { return smem_u32(&ctrl->low_full[x]); };
  const uint32_t b_qr = smem_u32(&ctrl->q_ready), b_sf = smem_u32(&ctrl->s_full), b_sx = smem_u32(&ctrl->s_free);
  const uint32_t b_pf = smem_u32(&ctrl->p_full), b_od = smem_u32(&ctrl->o_done), b_oe = smem_u32(&ctrl->o_empty);

  if (threadIdx.x == 0) {
    mbar_init(b_qr, 128);
    for (int x = 0; x < RT; ++x) {
      mbar_init(b_tf(x), FP8 ? kDcWiden : 1);  // fp8: the widening threads arrive
      mbar_init(b_te(x), 1);
      mbar_init(b_gf(x), 1);
      mbar_init(b_gr(x), 1);
      mbar_init(b_lf(x), kDcWiden);
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
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_kv);
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
        const int k0 = p.cu_k[dc_seq(p, s, sd.x).b];
        if (sg + 1 < seg_hi) {  // the next piece's query tokens (all heads), into L2
          const int bn = dc_seq(p, s, dc_seg(p, s, sg + 1).x).b;
          const int64_t q0n = p.cu_q[bn], rn = (p.cu_q[bn + 1] - q0n) * p.hq;
          if (rn > 0)
            tma_prefetch_bytes(reinterpret_cast<const uint16_t *>(p.q) + q0n * p.hq * kDcDqk,
                               (uint32_t)(rn * kDcDqk * 2));
        }
        for (int j = sd.y; ok && j < sd.z; ++j, ++tc) {
          const int x = tc % RT;
          if (!wait_bar<kDcColdReport>(b_te(x), ((tc / RT) & 1) ^ 1, abort_flag, hdr, kDSiteSlotEmpty, p.wait_ns)) {
            ok = false;
            break;
          }
          if (FP8) {  // the codes, into the upper half of the slot: chunks 0-2, then 3-8
            mbar_arrive_expect_tx(b_gf(x), kDcWidenLow * kDcStageChunkBytes);
            mbar_arrive_expect_tx(b_gr(x), (kDcChunks - kDcWidenLow) * kDcStageChunkBytes);
            for (int c = 0; c < kDcChunks; ++c)
              tma_load_2d(ring_u32 + x * kDcChunks * kDcChunkBytes + kDcStageOff + c * kDcStageChunkBytes, &tm_kv,
                          c < kDcWidenLow ? b_gf(x) : b_gr(x), c * 64, k0 + j * kDcKeys);
            // Tile j + 2 into L2, so that its load (issued once its slot is
            // free) does not wait on HBM: the widening adds to the time from
            // a free slot to a ready tile, which three slots must cover.
            if (j + 2 < sd.z)
              for (int c = 0; c < kDcChunks; ++c) tma_prefetch_2d(&tm_kv, c * 64, k0 + (j + 2) * kDcKeys);
          } else {
            mbar_arrive_expect_tx(b_tf(x), kDcChunks * kDcChunkBytes);
            for (int c = 0; c < kDcChunks; ++c)
              tma_load_2d(ring_u32 + (x * kDcChunks + c) * kDcChunkBytes, &tm_kv, b_tf(x), c * 64, k0 + j * kDcKeys);
          }
        }
      }
      // Teardown: every tile load this thread issued must have landed.
      const uint64_t t0 = global_ns();
      for (int x = 0; x < RT; ++x) {
        const uint32_t uses = tc / RT + ((uint32_t)x < tc % RT ? 1u : 0u);
        if (uses == 0) continue;
        while (!mbar_test(FP8 ? b_gf(x) : b_tf(x), (uses - 1) & 1) && global_ns() - t0 < p.wait_ns) {
        }
        while (FP8 && !mbar_test(b_gr(x), (uses - 1) & 1) && global_ns() - t0 < p.wait_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule, so MMA operands are computed
    // warp-uniformly; one elected lane issues each tcgen05 operation, and
    // the warp gives up a wait together if any lane gave up.
    const bool leader = elect_one();
    auto wait_warp = [&](uint32_t bar, uint32_t parity, volatile int *ab, WsHeader *h, uint32_t site) {
      return __all_sync(0xffffffffu, wait_bar<kDcColdReport>(bar, parity, ab, h, site, p.wait_ns));
    };
    {
      constexpr uint32_t idesc_s = make_idesc_f16(BF16, kDcRows, kDcKeys, false, false);
      constexpr uint32_t idesc_o = make_idesc_f16(BF16, kDcRows, 256, false, true);
      const uint32_t tmem_w = __shfl_sync(0xffffffffu, tmem, 0);
      const uint32_t s_tmem = tmem_w + (16u << 16);  // S chains and Q: lanes 16-31 of each sub-partition
      uint32_t tc = 0, g = 0, o_uses = 0;
      bool ok = true;
      // Descriptors: the high halves are fixed, a chunk / K-step only moves
      // the start address in the low half (16-byte units, never carries).
      const uint32_t k_hi = desc_hi(make_sdesc_sw128(ring_u32, 16, 1024));
      const uint32_t k_lo0 = desc_lo(make_sdesc_sw128(ring_u32, 16, 1024));
      const uint32_t v_hi = desc_hi(make_sdesc_sw128(ring_u32, kDcChunkBytes, 1024));
      const uint32_t v_lo0 = desc_lo(make_sdesc_sw128(ring_u32, kDcChunkBytes, 1024));
      const uint32_t p_hi = desc_hi(make_sdesc_sw128(p_u32, 16, 1024));
      const uint32_t p_lo0 = desc_lo(make_sdesc_sw128(p_u32, 16, 1024));
      // S of tile counter `t` into the three chains (chunk c accumulates into chain c % 3).
      auto issue_s = [&](uint32_t t) -> bool {
        const int x = t % RT;
        const uint32_t k_lo = k_lo0 + (uint32_t)((x * kDcChunks * kDcChunkBytes) >> 4);
        auto mma_chunk = [&](int c, int kk) {
          if (leader) mma_ts2(s_tmem + (c % 3) * kDcKeys, s_tmem + kDcQCol + (c * 4 + kk) * 8,
                  k_lo + (uint32_t)((c * kDcChunkBytes + kk * 32) >> 4), k_hi, idesc_s, (c >= 3 || kk > 0) ? 1u : 0u);
        };
        if (FP8) {
          // chunks 0-2 as soon as they are widened, then 3-8 (the first MMA
          // into each chain, c = 0, 1, 2 at kk = 0, still comes first)
          if (!wait_warp(b_lf(x), (t / RT) & 1, abort_flag, hdr, kDSiteSlotFull)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int c = 0; c < kDcWidenLow; ++c) mma_chunk(c, kk);
          if (!wait_warp(b_tf(x), (t / RT) & 1, abort_flag, hdr, kDSiteSlotFull)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int c = kDcWidenLow; c < kDcChunks; ++c) mma_chunk(c, kk);
        } else {
          if (!wait_warp(b_tf(x), (t / RT) & 1, abort_flag, hdr, kDSiteSlotFull)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int c = 0; c < kDcChunks; ++c) mma_chunk(c, kk);
        }
        if (leader) mma_commit(b_sf);
        return true;
      };
      for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
        const int4 sd = dc_seg(p, s, sg);
        const int n = sd.z - sd.y;
        if (!wait_warp(b_qr, (sg - seg_lo) & 1, abort_flag, hdr, kDSiteQReady)) break;
        tc_fence_after();
        if (g > 0 && !wait_warp(b_sx, (g - 1) & 1, abort_flag, hdr, kDSiteSFree)) break;
        if (!issue_s(tc)) break;
        for (int jj = 0; jj < n; ++jj, ++g, ++tc) {
          if (jj + 1 < n) {
            // the single S buffer is free once softmax has read S(g)
            if (!wait_warp(b_sx, g & 1, abort_flag, hdr, kDSiteSFree) || !issue_s(tc + 1)) {
              ok = false;
              break;
            }
          }
          if (!wait_warp(b_pf, g & 1, abort_flag, hdr, kDSitePFull)) {
            ok = false;
            break;
          }
          if (jj == 0 && o_uses > 0 && !wait_warp(b_oe, (o_uses - 1) & 1, abort_flag, hdr, kDSiteOEmpty)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_lo = v_lo0 + (uint32_t)(((tc % RT) * kDcChunks * kDcChunkBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int half = 0; half < 2; ++half)
              if (leader) mma_ss2(tmem_w + half * 256, p_lo0 + (uint32_t)(kk * 2), p_hi,
                      v_lo + (uint32_t)((half * 4 * kDcChunkBytes + kk * 16 * 128) >> 4), v_hi, idesc_o,
                      (jj > 0 || kk > 0) ? 1u : 0u);
          if (leader) mma_commit(b_od);
          if (leader) mma_commit(b_te(tc % RT));
        }
        ++o_uses;
      }
      if (leader) mma_commit(smem_u32(&ctrl->drain));
      const uint64_t t0 = global_ns();
      while (!mbar_test(smem_u32(&ctrl->drain), 0) && global_ns() - t0 < p.wait_ns) {
      }
    }
  } else if (FP8 && (warp >= 8 || warp == 2 || warp == 3)) {
    // ------------------------------------------------------------ fp8 -> bf16 widening (warps 8-11, 2-3)
    // Per tile 2,304 groups of 16 codes g = (chunk c, key row, u) = 256c +
    // 4 row + u: columns 16u..16u+15 of key `row` in chunk c, which become
    // 16-byte units 2u and 2u+1 of that row of bf16 chunk c, placed by the
    // 128B swizzle (unit ^ (row & 7)).  Widening thread t (0-191) takes
    // groups t + 192i: eight consecutive threads read 128 contiguous bytes
    // and write eight distinct units of two rows, so neither side has bank
    // conflicts.
    const int t = warp >= 8 ? threadIdx.x - 256 : threadIdx.x + 64;
    uint8_t *ring = smem_raw + (ring_u32 - smem_u32(smem_raw));
    auto put = [&](uint8_t *slot, int g, const uint4 &w) {
      const int c = g >> 8, row = (g >> 2) & 63, u = g & 3;
      uint4 a, b;
      e4m3x4_to_bf16x4(w.x, a.x, a.y);
      e4m3x4_to_bf16x4(w.y, a.z, a.w);
      e4m3x4_to_bf16x4(w.z, b.x, b.y);
      e4m3x4_to_bf16x4(w.w, b.z, b.w);
      uint8_t *drow = slot + c * kDcChunkBytes + row * 128;
      *reinterpret_cast<uint4 *>(drow + (((2 * u) ^ (row & 7)) << 4)) = a;
      *reinterpret_cast<uint4 *>(drow + (((2 * u + 1) ^ (row & 7)) << 4)) = b;
    };
    // The six warps give up a wait together (an AND over the widening
    // threads), so none of them is left waiting at a named barrier.
    auto agree = [&](bool got) {
      uint32_t all;
      asm volatile(
          "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
          : "=r"(all)
          : "r"(got ? 1u : 0u), "n"(kDcWiden)
          : "memory");
      return all != 0;
    };
    constexpr int kLow = kDcWidenLow * kDcKeys * 4 / kDcWiden;                   // groups per thread, chunks 0-2
    constexpr int kHigh = (kDcChunks - kDcWidenLow) * kDcKeys * 4 / kDcWiden;  // chunks 3-8
    uint32_t tc = 0;
    bool ok = true;
    for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
      const int4 sd = dc_seg(p, s, sg);
      for (int j = sd.y; j < sd.z; ++j, ++tc) {
        const int y = tc % RT;
        if (!agree(wait_bar<kDcColdReport>(b_gf(y), (tc / RT) & 1, abort_flag, hdr, kDSiteStageFull, p.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t *slot = ring + y * kDcChunks * kDcChunkBytes;
        const uint4 *codes = reinterpret_cast<const uint4 *>(slot + kDcStageOff);  // group g at codes[g]
        // chunks 0-2: their bf16 rows end below the codes
#pragma unroll
        for (int i = 0; i < kLow; ++i) put(slot, t + kDcWiden * i, codes[t + kDcWiden * i]);
        fence_proxy_async_smem();
        mbar_arrive(b_lf(y));  // S may start on chunks 0-2
        // chunks 3-8 (from chunk 4 on) overwrite codes: every thread reads
        // its groups (and has read its chunk 0-2 groups) before any write
        if (!agree(wait_bar<kDcColdReport>(b_gr(y), (tc / RT) & 1, abort_flag, hdr, kDSiteStageFull, p.wait_ns))) {
          ok = false;
          break;
        }
        constexpr int g0 = kDcWidenLow * kDcKeys * 4;
        uint4 w[kHigh];
#pragma unroll
        for (int i = 0; i < kHigh; ++i) w[i] = codes[g0 + t + kDcWiden * i];
        asm volatile("bar.sync 1, %0;" ::"n"(kDcWiden) : "memory");
#pragma unroll
        for (int i = 0; i < kHigh; ++i) put(slot, g0 + t + kDcWiden * i, w[i]);
        fence_proxy_async_smem();  // the MMA reads the chunks through the async proxy
        mbar_arrive(b_tf(y));
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax / epilogue
    const int sub = warp & 3, half = lane >> 4;
    const int r = sub * 16 + (lane & 15);                    // query row of this thread
    const uint32_t o_row = tmem + ((uint32_t)(sub * 32) << 16);
    const uint32_t s_row = tmem + ((uint32_t)(sub * 32 + 16) << 16);
    const float c = p.scale_log2;
    const bool neg = c < 0.f;
    const int G = p.hq / s.heads;  // query heads per sequence: row r is token r / G, head gh*G + r % G
    // Q rows of piece sg into TMEM (lanes 16-31, columns kDcQCol..): this
    // thread writes half `half` of row r; all global loads are issued first.
    auto load_q = [&](int sg) {
      const DcSeq sq_q = dc_seq(p, s, dc_seg(p, s, sg).x);
      const int bq = sq_q.b, ghq = sq_q.gh;
      const int q0 = p.cu_q[bq], rows = (p.cu_q[bq + 1] - q0) * G;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const uint16_t *>(p.q) + ((int64_t)(q0 + r / G) * p.hq + ghq * G + r % G) * kDcDqk);
      const bool vq = r < rows;
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        uint4 w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = vq ? src[(k2 * 2 + i / 8) * 16 + half * 8 + (i & 7)] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int k1 = 0; k1 < 2; ++k1) {
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 u = w[k1 * 8 + i];
            v[4 * i] = u.x; v[4 * i + 1] = u.y; v[4 * i + 2] = u.z; v[4 * i + 3] = u.w;
          }
          tmem_st_half32(s_row + kDcQCol + (k2 * 2 + k1) * 64, v);
        }
      }
      uint32_t v[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = vq ? src[64 + half * 4 + i] : make_uint4(0, 0, 0, 0);
        v[4 * i] = u.x; v[4 * i + 1] = u.y; v[4 * i + 2] = u.z; v[4 * i + 3] = u.w;
      }
      tmem_st_half16(s_row + kDcQCol + 256, v);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_qr);
    };
    uint32_t g = 0;
    bool ok = true;
    if (seg_lo < seg_hi) load_q(seg_lo);
    for (int sg = seg_lo; ok && sg < seg_hi; ++sg) {
      const int4 sd = dc_seg(p, s, sg);
      const DcSeq sq_v = dc_seq(p, s, sd.x);
      const int b = sq_v.b, gh = sq_v.gh;
      const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0, sk = p.cu_k[b + 1] - p.cu_k[b];
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
        uint32_t sv[32], sb[32];
        tmem_ld_half32(s_row + 0 * kDcKeys, sv);
        tmem_ld_half32(s_row + 1 * kDcKeys, sb);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[e] = __float_as_uint(__uint_as_float(sv[e]) + __uint_as_float(sb[e]));
        tmem_ld_half32(s_row + 2 * kDcKeys, sb);
        tc_fence_before();
        mbar_arrive(b_sx);  // S may be overwritten now
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[e] = __float_as_uint(__uint_as_float(sv[e]) + __uint_as_float(sb[e]));
        const int lim = nv - j * kDcKeys - half * 32;  // keys [0, lim) of this half are visible
        float ext = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = neg ? -__uint_as_float(sv[e]) : __uint_as_float(sv[e]);
          ext = (e < lim) ? fmaxf(ext, x) : ext;
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
        uint32_t pk[16];
        float rs = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0 = ex2(fmaf(__uint_as_float(sv[2 * e]), c, -base));
          float p1 = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), c, -base));
          p0 = (2 * e < lim) ? p0 : 0.f;
          p1 = (2 * e + 1 < lim) ? p1 : 0.f;
          rs += p0 + p1;
          pk[e] = BF16 ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
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
#pragma unroll 1
          for (int q = 0; q < kDcDv / 64; ++q) {
            uint32_t ov[32];
            tmem_ld_half32(o_row + q * 64, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st_half32(o_row + q * 64, ov);
          }
          tmem_wait_st();
        }
        // P row r, keys half*32 .. half*32+31: four 16-byte chunks, 128B swizzle.
        uint8_t *prow = p_gen + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = (half * 4 + i) ^ (r & 7);
          *reinterpret_cast<uint4 *>(prow + chunk * 16) = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
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
      const bool direct = dc_seg_cnt(p, s, sd.x) == 1;
      const int tok = q0 + (valid ? r / G : 0), h = gh * G + (valid ? r % G : 0);
      using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
      const float inv = l > 0.f ? (FP8 ? s.o_scale : 1.f) / l : 0.f;
#pragma unroll 1
      for (int q = 0; q < kDcDv / 64; ++q) {
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
          if (FP8) {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * s.o_scale);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *dc_pacc<kDcDv>(s, sg, r, col / 4 + e) = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
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
    // KV ring, drained above, is the scratch space)
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const int v = blockIdx.x / s.arith_k, i = blockIdx.x % s.arith_k, k = dc_seg_cnt(p, s, v);
    float *scratch = reinterpret_cast<float *>(smem_raw + kDcCtrlBytes);
    constexpr int NT = FP8 ? kDcThreadsFp8 : kDcThreads;
    if (k > 1 && i < k) dc_merge_pieces<T, kDcDv, NT>(p, s, v, i, k, scratch);
    else if (k == 0 && i == 0) dc_zero_rows<T, kDcDv, NT>(p, s, v);
  }
}

// ----------------------------------------------------------------------------
// Merge the pieces of every sequence that was split.  Row r of sequence
// v = (b, g) is query token r / G of batch entry b, head g*G + r % G, with
// G = Hq / heads.  One thread per (sequence v, 4-column group c4, row r) for
// r < R = min(64, max_q * G), rows fastest, so a warp's partial loads are
// contiguous; grid-stride.  Every unit is independent, so the dependent
// loads of all of them are in flight together.  A unit whose sequence was
// not split (stored directly by the decode kernel) costs one load, and when
// no sequence was split or left empty the kernel returns at once.
constexpr int kDcCombineThreads = 256;
constexpr int kDcCombineBatch = 4;  // pieces whose partials one thread loads in one round
template <typename T, int DV>
__global__ void __launch_bounds__(kDcCombineThreads) decode_combine_kernel(const AttnParams p, const DecodeSched s,
                                                                           int n_seq) {
  dc_pdl_wait();  // the decode kernel's partials
  if (*reinterpret_cast<volatile int *>(s.n_multi) == 0) return;
  constexpr int C4 = DV / 4;  // 4-column groups per row
  const int G = p.hq / s.heads;
  const int R = min(kDcRows, p.max_sq * G);
  const int64_t n_units = (int64_t)n_seq * C4 * R;
  for (int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; unit < n_units;
       unit += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(unit % R), c4 = (int)((unit / R) % C4), v = (int)(unit / ((int64_t)R * C4));
    // The sequence's piece count, first piece and query range are loaded in
    // one round, then (up to kDcCombineBatch pieces) every piece's (m, l) and
    // accumulator in a second one: the kernel's time is its chain of
    // dependent loads.  The sums run in piece order either way.
    const DcSeq sq = dc_seq(p, s, v);
    const int b = sq.b, gh = sq.gh;
    const int cnt = s.seg_cnt[v], base = s.seg_base[v];
    const int2 qr = dc_q(p, b);
    // not split: stored directly by the decode kernel (a sequence with no
    // piece, cnt = 0, is written here: O = 0, LSE = -inf)
    if (cnt == 1) continue;
    if (r >= qr.y * G) continue;
    float M = -INFINITY;
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto add = [&](float2 ml, float4 a) {
      const float w = ex2(ml.x - M);  // 0 for a piece that saw no visible key
      L += w * ml.y;
      acc.x = fmaf(w, a.x, acc.x);
      acc.y = fmaf(w, a.y, acc.y);
      acc.z = fmaf(w, a.z, acc.z);
      acc.w = fmaf(w, a.w, acc.w);
    };
    if (cnt <= kDcCombineBatch) {
      float2 ml[kDcCombineBatch];
      float4 a[kDcCombineBatch];
#pragma unroll
      for (int i = 0; i < kDcCombineBatch; ++i)
        if (i < cnt) {
          ml[i] = s.part_ml[(int64_t)(base + i) * kDcRows + r];
          a[i] = *dc_pacc<DV>(s, base + i, r, c4);
        }
#pragma unroll
      for (int i = 0; i < kDcCombineBatch; ++i)
        if (i < cnt) M = fmaxf(M, ml[i].x);
      if (M != -INFINITY) {
#pragma unroll
        for (int i = 0; i < kDcCombineBatch; ++i)
          if (i < cnt) add(ml[i], a[i]);
      }
    } else {
      for (int i = 0; i < cnt; ++i) M = fmaxf(M, s.part_ml[(int64_t)(base + i) * kDcRows + r].x);
      if (M != -INFINITY) {
#pragma unroll 4
        for (int i = 0; i < cnt; ++i) add(s.part_ml[(int64_t)(base + i) * kDcRows + r], *dc_pacc<DV>(s, base + i, r, c4));
      }
    }
    const int tok = qr.x + r / G, h = gh * G + r % G;
    T *orow = reinterpret_cast<T *>(p.o) + (int64_t)tok * p.o_rs + (int64_t)h * p.o_hs + 4 * c4;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    dc_store4<T>(orow, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (c4 == 0 && p.lse)
      p.lse[(int64_t)tok * p.hq + h] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace mxfa
