// route_permute_combine.cuh -- the memory-light steps of the routed-expert
// layer: top-k routing, grouping by expert, weighted combine, and the
// group-128 quantiser used to build INT8/INT4 experts.
//
// All follow "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
// Inference": routing equation of Section 3.1, grouping of Figure 1, combine of
// Section 3.4, quantiser equation of Section 3.2.
#pragma once

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------ routing --

// Orderable key of a logit: larger key <=> larger value, -0.0 and +0.0 share a
// key, NaN takes the key of -inf.  Every real key is >= 0x007FFFFF, so 0 marks
// an empty slot.
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of one token by one warp.  Lane l holds the keys of experts l, l+32,
// ... (KEYS slots, ascending id).  k rounds of warp argmax pick the experts by
// descending logit, ties to the lowest id; lane j < k returns the j-th pick
// and its gating weight.  nan_seen: some logit of the token was NaN (warp-wide).
template <int KEYS>
__device__ __forceinline__ void route_token(const float* __restrict__ z, int E, int k,
                                            int renormalize, int lane, int& pick_e,
                                            float& pick_w, bool& nan_seen) {
  uint32_t key[KEYS];
  bool nan_here = false;
#pragma unroll
  for (int i = 0; i < KEYS; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < E) {
      float v = z[e];
      if (isnan(v)) {
        nan_here = true;
        v = -INFINITY;
      }
      key[i] = logit_key(v);
    }
  }
  nan_seen = __any_sync(0xffffffffu, nan_here);

  int my_e = 0;
  float my_z = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0;
    int best_i = -1;
#pragma unroll
    for (int i = 0; i < KEYS; ++i)
      if (key[i] > best) {  // strict: the lowest id among this lane's equal keys
        best = key[i];
        best_i = i;
      }
    const uint32_t win_key = __reduce_max_sync(0xffffffffu, best);
    const uint32_t cand =
        (best_i >= 0 && best == win_key) ? (uint32_t)(lane + 32 * best_i) : 0xffffffffu;
    const uint32_t win_e = __reduce_min_sync(0xffffffffu, cand);
    if ((int)(win_e & 31) == lane) {
#pragma unroll
      for (int i = 0; i < KEYS; ++i)
        if (i == (int)(win_e >> 5)) key[i] = 0;
    }
    if (lane == j) {
      my_e = (int)win_e;
      my_z = key_logit(win_key);
    }
  }

  // Gating weights.  m = the largest selected logit (pick 0).
  const float m = __shfl_sync(0xffffffffu, my_z, 0);
  const float ex = (lane < k) ? expf(my_z - m) : 0.0f;
  float den = 0.0f;
  if (renormalize) {
    for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, ex, j);
  } else {
    float part = 0.0f;
    for (int e = lane; e < E; e += 32) {
      const float v = z[e];
      if (!isnan(v)) part += expf(v - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    den = part;
  }
  pick_e = my_e;
  pick_w = ex / den;
}

// One warp per token.
template <int KEYS>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T,
                                                         int E, int k, int renormalize,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_w) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int e;
  float w;
  bool nan_seen;
  route_token<KEYS>(logits + (size_t)t * E, E, k, renormalize, lane, e, w, nan_seen);
  if (nan_seen && lane == 0) flag_status(MOE_STATUS_NONFINITE_LOGIT);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = e;
    topk_w[(size_t)t * k + lane] = w;
  }
}

// -------------------------------------------------------------- permutation --

constexpr int kPermuteThreads = 1024;
constexpr int kPermuteWarps = kPermuteThreads / 32;

constexpr int kPermuteChunk = 256;   // tokens per CTA when the grouping is split over CTAs

__host__ __device__ constexpr size_t permute_smem_bytes(int E) {
  return (size_t)(2 * kPermuteWarps + 2) * E * sizeof(int32_t);
}

// Large batches, first pass: CTA b counts the valid pairs of tokens
// [b * kPermuteChunk, (b + 1) * kPermuteChunk) per expert into
// blk_counts[b * E + e] (the same validity rule as permute_index_kernel).
__global__ void __launch_bounds__(kPermuteThreads)
    permute_count_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                         int32_t* __restrict__ blk_counts) {
  extern __shared__ int32_t cnt[];
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kPermuteChunk, t1 = min(T, t0 + kPermuteChunk);
  for (int t = t0 + tid; t < t1; t += blockDim.x) {
    int ev[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) ev[j] = (j < k) ? idx[(size_t)t * k + j] : -1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= k) break;
      bool ok = ev[j] >= 0 && ev[j] < E;
#pragma unroll
      for (int jj = 0; jj < j; ++jj) ok = ok && (ev[jj] != ev[j]);
      if (ok) atomicAdd(&cnt[ev[j]], 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) blk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// Grouping of tokens [c0, c1) by one CTA; warp w owns a contiguous chunk.
//   1. per-(warp, expert) counts (shared-memory atomics: order-free sums)
//   2. exclusive scan over (expert, warp) -> expert_offsets and per-warp bases
//   3. each warp walks its tokens 32 at a time in token order; a token's rank
//      inside expert e is the number of lower lanes that also chose e, read
//      from a per-(warp, expert) lane bitmask.
// One CTA (blk_counts == nullptr): c0 = 0, c1 = T.  Split over CTAs: CTA b
// takes tokens [b * kPermuteChunk, ...) and adds, per expert, the pairs of all
// experts below and of the CTAs before it (from permute_count_kernel), so the
// result is the same.  The order (expert id, then token) is fixed; no atomic
// decides it.
__global__ void __launch_bounds__(kPermuteThreads, 1)
    permute_index_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                         int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
                         int32_t* __restrict__ dest_row,
                         const int32_t* __restrict__ blk_counts,
                         unsigned int* __restrict__ hot) {
  extern __shared__ int32_t psm[];
  int32_t* base = psm;                                          // [warps][E]
  uint32_t* mask = reinterpret_cast<uint32_t*>(psm + kPermuteWarps * E);  // [warps][E]
  int32_t* tot = psm + 2 * kPermuteWarps * E;                   // [E]
  int32_t* pre = tot + E;                                       // [E] pairs of earlier CTAs
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool split = blk_counts != nullptr;
  const bool lead = !split || blockIdx.x == 0;
  pdl_launch_dependents();
  pdl_wait();

  for (int i = tid; i < 2 * kPermuteWarps * E; i += blockDim.x) psm[i] = 0;
  __syncthreads();

  const int c0 = split ? (int)blockIdx.x * kPermuteChunk : 0;
  const int c1 = split ? min(T, c0 + kPermuteChunk) : T;
  const int chunk = (c1 - c0 + kPermuteWarps - 1) / kPermuteWarps;
  const int t_begin = min(c1, c0 + warp * chunk);
  const int t_end = min(c1, t_begin + chunk);

  // 1. counts of the valid pairs
  bool bad = false;
  for (int t = t_begin + lane; t < t_end; t += 32) {
    int ev[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) ev[j] = (j < k) ? idx[(size_t)t * k + j] : -1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= k) break;
      bool ok = ev[j] >= 0 && ev[j] < E;
#pragma unroll
      for (int jj = 0; jj < j; ++jj) ok = ok && (ev[jj] != ev[j]);
      if (ok)
        atomicAdd(&base[warp * E + ev[j]], 1);
      else
        bad = true;
    }
  }
  if (bad) flag_status(MOE_STATUS_BAD_EXPERT_ID);
  __syncthreads();

  // 2a. per expert, exclusive prefix over warps; tot = this CTA's pairs, or
  // with the split, all CTAs' pairs (pre = those of the CTAs before this one)
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kPermuteWarps; ++w) {
      const int c = base[w * E + e];
      base[w * E + e] = run;
      run += c;
    }
    tot[e] = run;
    if (split) {
      int all = 0, before = 0;
      for (int b = 0; b < (int)gridDim.x; ++b) {
        const int c = blk_counts[(size_t)b * E + e];
        all += c;
        if (b < (int)blockIdx.x) before += c;
      }
      tot[e] = all;
      pre[e] = before;
    }
  }
  __syncthreads();
  // 2b. exclusive scan of the expert totals (warp 0; lane owns a run of ids)
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (e0 + i < E) local += tot[e0 + i];
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        const int c = tot[e];
        tot[e] = run + (split ? pre[e] : 0);
        if (lead) offsets[e] = run;
        if (lead && hot != nullptr && c != 0) atomicAdd(hot + e, (unsigned int)c);
        run += c;
      }
    }
    if (lead && lane == 31) offsets[E] = incl;
  }
  __syncthreads();
  for (int i = tid; i < kPermuteWarps * E; i += blockDim.x) base[i] += tot[i % E];
  __syncthreads();

  // 3. stable scatter
  int32_t* wbase = base + warp * E;
  uint32_t* wmask = mask + warp * E;
  const uint32_t lower = (1u << lane) - 1u;
  for (int tb = t_begin; tb < t_end; tb += 32) {
    const int t = tb + lane;
    const bool tv = t < t_end;
    int ev[16];
    bool ok[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ev[j] = (tv && j < k) ? idx[(size_t)t * k + j] : -1;
      ok[j] = ev[j] >= 0 && ev[j] < E;
#pragma unroll
      for (int jj = 0; jj < j; ++jj) ok[j] = ok[j] && (ev[jj] != ev[j]);
      if (ok[j]) atomicOr(&wmask[ev[j]], 1u << lane);
    }
    __syncwarp();
    uint32_t mm[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      mm[j] = 0;
      if (ok[j]) {
        mm[j] = wmask[ev[j]];
        const int row = wbase[ev[j]] + __popc(mm[j] & lower);
        dest_row[(size_t)t * k + j] = row;
        perm_token[row] = t;
      } else if (tv && j < k) {
        dest_row[(size_t)t * k + j] = -1;
      }
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (ok[j] && (mm[j] & lower) == 0) {  // lowest lane of this expert updates
        wbase[ev[j]] += __popc(mm[j]);
        wmask[ev[j]] = 0;
      }
    __syncwarp();
  }
}

// x_perm[r] = x[perm_token[r]] for r < offsets[E], 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm_token,
                                                          const int32_t* __restrict__ offsets,
                                                          int E, int vec_per_row,
                                                          uint4* __restrict__ x_perm) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = (size_t)offsets[E] * vec_per_row;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / vec_per_row, c = i % vec_per_row;
    x_perm[i] = x[(size_t)perm_token[r] * vec_per_row + c];
  }
}

// ------------------------------------------- routing + grouping, small batch --

constexpr int kFrontThreads = 1024;
constexpr int kFrontMaxTokens = 128;

__host__ __device__ constexpr size_t front_smem_bytes(int T, int k, int E) {
  return (size_t)2 * T * k * sizeof(int32_t) + (size_t)2 * E * sizeof(int32_t);
}

// Routing, grouping and the row gather of a small batch (T <= 128) in one
// launch, with the same results as route_topk_kernel + permute_index_kernel +
// gather_rows_kernel.  Every CTA routes all T tokens into shared memory (a few
// KB of logits) and derives the whole permutation, so no CTA waits for
// another; CTA b then copies rows b, b + G, ... of x_perm, and CTA 0 alone
// writes the index outputs and zeroes `zero_n` ints at `zero_ptr` (the FFN's
// scheduler counters: after griddepcontrol.wait, so every earlier use of them
// is complete).  Ids come from the routing above, so all are valid and
// distinct within a token.
template <int KEYS>
__global__ void __launch_bounds__(kFrontThreads, 1)
    route_permute_gather_kernel(const float* __restrict__ logits, const uint4* __restrict__ x,
                                int T, int E, int k, int renormalize, int vec_per_row,
                                int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
                                int32_t* __restrict__ dest_row, uint4* __restrict__ x_perm,
                                int* __restrict__ zero_ptr, int zero_n,
                                unsigned int* __restrict__ hot) {
  extern __shared__ int32_t fsm[];
  const int pairs = T * k;
  int32_t* sidx = fsm;                                     // [pairs] expert of pair (t, j)
  int32_t* sperm = sidx + pairs;                           // [pairs] token of permuted row
  int32_t* base = sperm + pairs;                           // [E]
  uint32_t* mask = reinterpret_cast<uint32_t*>(base + E);  // [E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool lead = blockIdx.x == 0;
  pdl_launch_dependents();
  pdl_wait();

  if (lead)
    for (int i = tid; i < zero_n; i += blockDim.x) zero_ptr[i] = 0;
  for (int i = tid; i < 2 * E; i += blockDim.x) base[i] = 0;  // base and mask

  // 1. top-k: warp w routes tokens w, w + 32, ...
  for (int t = warp; t < T; t += kFrontThreads / 32) {
    int e;
    float w;
    bool nan_seen;
    route_token<KEYS>(logits + (size_t)t * E, E, k, renormalize, lane, e, w, nan_seen);
    if (lane < k) {
      sidx[t * k + lane] = e;
      if (lead) {
        topk_idx[(size_t)t * k + lane] = e;
        topk_w[(size_t)t * k + lane] = w;
      }
    }
    if (lead && nan_seen && lane == 0) flag_status(MOE_STATUS_NONFINITE_LOGIT);
  }
  __syncthreads();

  // 2. counts, exclusive scan, stable ranks (warp 0; order = expert id, then token)
  if (warp == 0) {
    for (int i = lane; i < pairs; i += 32) atomicAdd(&base[sidx[i]], 1);
    __syncwarp();
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (e0 + i < E) local += base[e0 + i];
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        const int c = base[e];
        base[e] = run;
        if (lead) offsets[e] = run;
        if (lead && hot != nullptr && c != 0) atomicAdd(hot + e, (unsigned int)c);
        run += c;
      }
    }
    if (lead && lane == 31) offsets[E] = incl;
    __syncwarp();
    const uint32_t lower = (1u << lane) - 1u;
    for (int tb = 0; tb < T; tb += 32) {  // lane = token tb + lane
      const int t = tb + lane;
      const bool tv = t < T;
      for (int j = 0; j < k; ++j)
        if (tv) atomicOr(&mask[sidx[t * k + j]], 1u << lane);
      __syncwarp();
      // Every lane reads the masks of all its experts before any lane updates
      // base/mask (the __syncwarp between the two loops), so the update never
      // depends on how the lanes' j iterations interleave.
      int ev[16];
      uint32_t mm[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ev[j] = -1;
        mm[j] = 0;
        if (tv && j < k) {
          ev[j] = sidx[t * k + j];
          mm[j] = mask[ev[j]];
          const int row = base[ev[j]] + __popc(mm[j] & lower);
          sperm[row] = t;
          if (lead) {
            dest_row[(size_t)t * k + j] = row;
            perm_token[row] = t;
          }
        }
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (ev[j] >= 0 && (mm[j] & lower) == 0) {  // lowest lane of this expert updates
          base[ev[j]] += __popc(mm[j]);
          mask[ev[j]] = 0;
        }
      __syncwarp();
    }
  }
  __syncthreads();

  // 3. this CTA's rows of x_perm
  const int G = gridDim.x;
  const int rows_here = (pairs - (int)blockIdx.x + G - 1) / G;
  for (int i = tid; i < rows_here * vec_per_row; i += blockDim.x) {
    const int r = (int)blockIdx.x + (i / vec_per_row) * G, c = i % vec_per_row;
    x_perm[(size_t)r * vec_per_row + c] = x[(size_t)sperm[r] * vec_per_row + c];
  }
}

// ------------------------------------------------------------------ combine --

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// out[t] = sum_j w[t][j] * y[dest_row[t][j]] in fp32, j = 0..k-1 in order.
// grid (T, ceil(H/8 / blockDim.x)); each thread one 16-byte vector of a row.
// Pairs with dest_row < 0 are skipped; a row >= rows (the capacity of y,
// T * k) is skipped too and flagged, so no read leaves y.
// The k row indices and weights are loaded first, then all k vectors, and only
// then summed (same order as above): two dependent memory round trips per
// token instead of k, which at decode sizes is most of the kernel's time.
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y,
                                                      const int32_t* __restrict__ dest_row,
                                                      const float* __restrict__ topk_w, int k,
                                                      int vec_per_row, int rows,
                                                      uint4* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= vec_per_row) return;
  constexpr int kMaxK = 16;  // the host rejects k > 16
  int r[kMaxK];
  float wt[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    r[j] = -1;
    wt[j] = 0.0f;
    if (j < k) {
      r[j] = dest_row[(size_t)t * k + j];
      wt[j] = topk_w[(size_t)t * k + j];
    }
  }
  uint4 v[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    v[j] = make_uint4(0u, 0u, 0u, 0u);
    if (r[j] >= 0 && r[j] < rows) v[j] = y[(size_t)r[j] * vec_per_row + c];
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (r[j] < 0) continue;
    if (r[j] >= rows) {
      if (c == 0) flag_status(MOE_STATUS_BAD_ROW_INDEX);
      continue;
    }
    float f[8];
    bf16x8_to_f32(v[j], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(wt[j], f[i], acc[i]);
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  out[(size_t)t * vec_per_row + c] = o;
}

// ---------------------------------------------------------------- quantiser --

// One warp per (row, K-group of 128); lane holds 4 consecutive elements.
// s = fp16_rne(amax / Q) (binary32 quotient), q = clip(rint_even(W / s)).
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ w, int rows,
                                                       int K, int prec, uint8_t* __restrict__ q,
                                                       uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int groups = K / 128;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (gw >= (long long)rows * groups) return;
  const int row = (int)(gw / groups), g = (int)(gw % groups);
  const uint2 raw = *reinterpret_cast<const uint2*>(w + (size_t)row * K + g * 128 + lane * 4);
  float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  uint32_t amax_bits = 0;  // |v| as non-negative float bits order like the values
#pragma unroll
  for (int i = 0; i < 4; ++i) amax_bits = max(amax_bits, __float_as_uint(fabsf(v[i])));
  amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
  const int Q = (prec == MOE_INT4) ? 7 : 127;
  const __half sh = __float2half_rn(__fdiv_rn(__uint_as_float(amax_bits), (float)Q));
  const float s = __half2float(sh);
  int qv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int c = 0;
    if (s != 0.0f) c = __float2int_rn(__fdiv_rn(v[i], s));
    qv[i] = min(Q, max(-Q - 1, c));
  }
  if (lane == 0) scales[(size_t)g * rows + row] = __half_as_ushort(sh);
  if (prec == MOE_INT8) {
    const uint32_t packed = (uint32_t)(qv[0] & 0xFF) | ((uint32_t)(qv[1] & 0xFF) << 8) |
                            ((uint32_t)(qv[2] & 0xFF) << 16) | ((uint32_t)(qv[3] & 0xFF) << 24);
    *reinterpret_cast<uint32_t*>(q + (size_t)row * K + g * 128 + lane * 4) = packed;
  } else {
    const uint16_t packed = (uint16_t)((qv[0] + 8) | ((qv[1] + 8) << 4) | ((qv[2] + 8) << 8) |
                                       ((qv[3] + 8) << 12));
    *reinterpret_cast<uint16_t*>(q + (size_t)row * (K / 2) + g * 64 + lane * 2) = packed;
  }
}

// ----------------------------------------------------------- hot experts --
// Hot set of one layer (DynaExq abstract: a per-layer set of hot experts,
// estimated from router traces, under a memory budget): the n experts with the
// highest selection counts, ties to the lower id, written in ascending id
// order.  One CTA, one thread per expert (E <= 512): an expert's rank is the
// number of experts before it in (count descending, id ascending) order, found
// by comparing with every count; its output slot is the number of selected
// experts with a lower id.  zero != 0 clears the counts afterwards (a new
// counting window starts).
constexpr int kSelectThreads = 512;

__global__ void __launch_bounds__(kSelectThreads)
    select_hot_kernel(unsigned int* __restrict__ counts, int E, int n, int zero,
                      int32_t* __restrict__ hot_ids) {
  __shared__ unsigned int c[kSelectThreads];
  __shared__ int sel[kSelectThreads];
  const int e = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  c[e] = e < E ? counts[e] : 0u;
  __syncthreads();
  int rank = 0;
  if (e < E) {
    const unsigned int mine = c[e];
    for (int j = 0; j < E; ++j) rank += (c[j] > mine) || (c[j] == mine && j < e);
  }
  sel[e] = (e < E && rank < n) ? 1 : 0;
  __syncthreads();
  if (sel[e]) {
    int pos = 0;
    for (int j = 0; j < e; ++j) pos += sel[j];
    hot_ids[pos] = e;
  }
  if (zero && e < E) counts[e] = 0u;
}

}  // namespace moe
