// sched.cuh -- device-side schedule for the varlen tensor-core prefill.
//
// The host never sees the sequence lengths (cu_seqlens live on the device
// and no call synchronises), so one small CTA builds the work list on the
// stream right before the attention kernel: every (sequence b, 256-row
// query block m) pair, ordered by decreasing number of KV tiles (largest
// causal blocks first, so the persistent CTAs finish close together), by a
// counting sort over the tile count.
#pragma once

#include <cub/block/block_scan.cuh>

#include "prefill_tc.cuh"

namespace mxfa {

constexpr int kPrepThreads = 1024;

__device__ __forceinline__ int pair_cost(const AttnParams &p, int b, int m) {
  const SeqRange sr = seq_range(p, b);
  int cost = 0;
  for (int t = 0; t < 2; ++t) {
    const int first = m * kTcUnitRows + t * kTcBlockM;
    if (first < sr.sq) {
      const int last = min(sr.sq - 1, first + kTcBlockM - 1);
      cost += (visible_keys(last, sr.sq, sr.sk, p.causal) + kTcBlockN - 1) / kTcBlockN;
    }
  }
  return cost;
}

// Largest b with prefix[b] <= idx.
__device__ __forceinline__ int find_block_seq(const int *prefix, int batch, int idx) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// prefix: [batch + 1] ints, bucket: [n_buckets] ints, pairs: [max_pairs].
__global__ void __launch_bounds__(kPrepThreads)
prefill_prep_kernel(const AttnParams p, int *prefix, int *bucket, int n_buckets, int2 *pairs, int max_pairs) {
  using Scan = cub::BlockScan<int, kPrepThreads>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int carry, n_blocks;
  const int tid = threadIdx.x;
  if (tid == 0) carry = 0;
  for (int i = tid; i < n_buckets; i += kPrepThreads) bucket[i] = 0;
  __syncthreads();

  // prefix[b] = number of 256-row blocks in sequences < b
  for (int base = 0; base < p.batch; base += kPrepThreads) {
    const int b = base + tid;
    int x = 0;
    if (b < p.batch) x = (p.cu_q[b + 1] - p.cu_q[b] + kTcUnitRows - 1) / kTcUnitRows;
    int incl, total;
    Scan(tmp).InclusiveSum(x, incl, total);
    if (b < p.batch) prefix[b + 1] = carry + incl;
    __syncthreads();
    if (tid == 0) carry += total;
    __syncthreads();
  }
  if (tid == 0) {
    prefix[0] = 0;
    n_blocks = carry;  // every (sequence, 256-row block) pair, before the clamp to the schedule's room
  }
  __syncthreads();
  const int n_pairs = min(n_blocks, max_pairs);

  // histogram over key = (n_buckets - 1 - cost): descending cost
  for (int idx = tid; idx < n_pairs; idx += kPrepThreads) {
    const int b = find_block_seq(prefix, p.batch, idx);
    const int key = max(0, n_buckets - 1 - pair_cost(p, b, idx - prefix[b]));
    atomicAdd(&bucket[key], 1);
  }
  __syncthreads();
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_buckets; base += kPrepThreads) {
    const int i = base + tid;
    const int x = i < n_buckets ? bucket[i] : 0;
    int excl, total;
    Scan(tmp).ExclusiveSum(x, excl, total);
    __syncthreads();
    if (i < n_buckets) bucket[i] = carry + excl;
    __syncthreads();
    if (tid == 0) carry += total;
    __syncthreads();
  }
  for (int idx = tid; idx < n_pairs; idx += kPrepThreads) {
    const int b = find_block_seq(prefix, p.batch, idx);
    const int m = idx - prefix[b];
    const int key = max(0, n_buckets - 1 - pair_cost(p, b, m));
    const int pos = atomicAdd(&bucket[key], 1);
    pairs[pos] = make_int2(b, m);
  }
  if (tid == 0) {
    p.hdr->n_units = (uint32_t)n_pairs;
    // A sequence longer than the max_seqlen_q the schedule was sized for
    // leaves blocks unscheduled: their rows of O would never be written.
    if (n_blocks > max_pairs) report_error(p.hdr, 1u /* MXFA_ERR_INVALID_ARG */, 0x201);
  }
}

}  // namespace mxfa
