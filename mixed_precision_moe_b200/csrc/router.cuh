// router.cuh -- the router projection fused with top-k routing.
//
// "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference",
// Section 3.1 routing equation: z_t = W_r h_t, S_t = TopK(z_t, k); the router
// stays in BF16 (Abstract).  Here h (bf16 [T][H]) and W_r (bf16 [E][H]) are
// multiplied on the tensor cores with fp32 accumulation, and the fp32 logits
// feed the same warp top-k and gating weights as route_topk_kernel.
//
// Layout of the work.  A tile is `tm` tokens (128; 64 when E > 256, so that a
// tile's partial logits fit in shared memory) times all E experts (N = E
// rounded up to 16, at most 512: one or two MMAs of N <= 256 per K step).  The
// K (hidden) dimension of a tile is split over the S CTAs of a thread-block
// cluster; each CTA accumulates its K slice in TMEM, stages the partial
// logits in its shared memory, and after a cluster barrier CTA s sums the S
// partials of its share of the tile's rows over distributed shared memory in
// the fixed order 0 .. S-1 (deterministic, no atomics), writes the logits and
// routes those tokens.  Token rows beyond T are zero-filled by TMA; expert
// rows beyond E give zero columns that the top-k never reads.
#pragma once

#include "common.cuh"
#include "route_permute_combine.cuh"

namespace moe {
namespace router {

constexpr int kThreads = 512;     // 16 warps; warp w reads TMEM lane quadrant w % 4
constexpr int kKB = 64;           // K-elements per stage: one 128-byte swizzled row
constexpr int kMaxE = 512;
constexpr int kMaxCluster = 16;   // non-portable cluster size (8 is portable)
constexpr uint32_t kHStage = 16384;   // 128 rows x 128 B (M = 128 reads all of it)
constexpr uint32_t kWChunk = 32768;   // 256 expert rows x 128 B
constexpr size_t kSmemLimit = 227 * 1024;

struct Params {
  int T, H, E, k, renormalize, do_topk;
  int npad;   // E rounded up to 16
  int tm;     // token rows per tile
  int hrows;  // rows per h copy: min(tm, T rounded up to 8); the MMA's other A rows are unused
  int nkb;    // H / kKB
  int ns;     // ring stages
  float* logits;       // [T][E] or null
  int32_t* topk_idx;   // [T][k] (do_topk)
  float* topk_w;       // [T][k] (do_topk)
};

__host__ __device__ constexpr int npad_of(int E) { return (E + 15) & ~15; }
__host__ __device__ constexpr int tm_of(int E) { return npad_of(E) > 256 ? 64 : 128; }
__host__ __device__ constexpr uint32_t wstage_of(int npad) {
  return npad > 256 ? 2 * kWChunk : (uint32_t)npad * 128u;
}
__host__ __device__ constexpr uint32_t tmem_cols_of(int npad) {
  return npad <= 32 ? 32 : npad <= 64 ? 64 : npad <= 128 ? 128 : npad <= 256 ? 256 : 512;
}

// Shared memory, from a 1024-byte aligned base (the same offsets in every CTA
// of the cluster):
//   [0, ring)   ns stages of {h tile (16 KB), W_r tile}; after the MMAs the
//               same bytes hold the partial logits [tm][npad + 4] fp32 (the
//               4-float pad makes the row-per-thread stores conflict-free)
//   zbuf        the reduced logits of this CTA's rows [rpc][npad] (S > 1)
//   bar         full[ns], empty[ns], done
//   misc        TMEM address, abort flag
struct Layout {
  uint32_t ring, zbuf, bar, misc, total;
};

__host__ __device__ inline Layout layout(int npad, int tm, int ns, int S) {
  Layout L;
  const uint32_t stage = kHStage + wstage_of(npad);
  const uint32_t part = (uint32_t)tm * (npad + 4) * 4u;
  L.ring = ((ns * stage > part ? ns * stage : part) + 1023u) & ~1023u;
  const int rpc = (tm + S - 1) / S;
  L.zbuf = L.ring;
  const uint32_t zbytes = S > 1 ? (uint32_t)rpc * npad * 4u : 0u;
  L.bar = (L.zbuf + zbytes + 15u) & ~15u;
  L.misc = L.bar + (2 * ns + 1) * 8;
  L.total = L.misc + 16 + 1024;  // + alignment slack of the dynamic base
  return L;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_nctas() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Barrier over every thread of the cluster; release/acquire orders the
// shared-memory writes before it with the peers' reads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Grid (S, tiles), cluster (S, 1, 1), S <= 16.  Warp 0 lane 0 issues the TMA copies,
// warp 1 lane 0 the MMAs; then all 16 warps drain the accumulator (warp w
// reads TMEM lanes 32 (w % 4) .. + 31 = tile rows, every fourth 16-column
// chunk), reduce and route: the top-k's dependent warp reductions need many
// warps in flight.  Every wait is bounded;
// a thread that gives up sets MOE_STATUS_WAIT_TIMEOUT and still takes part in
// both cluster barriers, so no CTA waits for one that left.
template <int KEYS>
__global__ void __launch_bounds__(kThreads, 1)
    router_topk_kernel(const __grid_constant__ CUtensorMap tm_h,
                       const __grid_constant__ CUtensorMap tm_w, const Params p) {
  extern __shared__ uint8_t rt_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = (int)cluster_nctas();
  const int s = (int)cluster_rank();
  const Layout L = layout(p.npad, p.tm, p.ns, S);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bar);
  uint64_t* empty = full + p.ns;
  uint64_t* done = empty + p.ns;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t stage = kHStage + wstage_of(p.npad);
  const uint32_t ncols = tmem_cols_of(p.npad);
  const int row0 = blockIdx.y * p.tm;
  const int rows = min(p.tm, p.T - row0);
  const int kb0 = s * p.nkb / S, nkl = (s + 1) * p.nkb / S - kb0;
  const int nchunk = p.npad > 256 ? 2 : 1;

  // Thread 0 initialises the barriers and, as the producer, issues the copies
  // of the first ns stages at once (they need no free stage), overlapping the
  // TMEM allocation and the block-wide sync that publishes it.
  const uint32_t tx = (uint32_t)p.hrows * 128u + wstage_of(p.npad);
  auto issue = [&](int i) {
    const int st = i % p.ns;
    uint8_t* hs = base + st * stage;
    uint8_t* ws = hs + kHStage;
    const int kx = (kb0 + i) * kKB;
    mbar_arrive_expect_tx(&full[st], tx);
    tma_load_2d(hs, &tm_h, kx, row0, &full[st]);
    for (int c = 0; c < nchunk; ++c) tma_load_2d(ws + c * kWChunk, &tm_w, kx, c * 256, &full[st]);
  };
  const int first = min(nkl, p.ns);
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_h);
    prefetch_tmap(&tm_w);
    pdl_wait();  // h may come from the previous kernel in the stream
    for (int i = 0; i < first; ++i) issue(i);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------- producer: the stages beyond ns
    int issued = first;
    for (int i = first; i < nkl; ++i) {
      const int st = i % p.ns;
      if (!mbar_wait(&empty[st], ((i / p.ns) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      issue(i);
      issued = i + 1;
    }
    if (*abort_flag) {  // let the copies in flight land before the bytes are reused
      for (int i = max(0, issued - p.ns); i < issued; ++i)
        mbar_wait(&full[i % p.ns], (i / p.ns) & 1, nullptr, 2000000ll);
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------------- MMA
    const uint64_t hdesc0 = smem_desc_sw128(smem_u32(base));
    const uint64_t wdesc0 = smem_desc_sw128(smem_u32(base + kHStage));
    const uint32_t sstep = stage >> 4, cstep = kWChunk >> 4;
    const uint32_t id0 = idesc_bf16_f32(128, nchunk == 2 ? 256 : p.npad);
    const uint32_t id1 = idesc_bf16_f32(128, nchunk == 2 ? p.npad - 256 : 16);
    for (int i = 0; i < nkl; ++i) {
      const int st = i % p.ns;
      if (!mbar_wait(&full[st], (i / p.ns) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint64_t hd = hdesc0 + st * sstep, wd = wdesc0 + st * sstep;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (i | kk) != 0;
        mma_bf16_ss(tmem, hd + 2 * kk, wd + 2 * kk, id0, acc);
        if (nchunk == 2) mma_bf16_ss(tmem + 256, hd + 2 * kk, wd + cstep + 2 * kk, id1, acc);
      }
      mma_commit(&empty[st]);
    }
    mma_commit(done);  // arrives once every MMA issued above has completed
  }

  // ------------------------------------------------ accumulator -> partials
  __syncwarp();
  bool ok = mbar_wait(done, 0, abort_flag) && !*abort_flag;
  tc_fence_after();
  __syncwarp();
  const int pstride = p.npad + 4;
  float* part = reinterpret_cast<float*>(base);
  const int quad = warp & 3, r = quad * 32 + lane;
  // the four warps of a lane quadrant take every fourth 16-column chunk
  for (int c = (warp >> 2) * 16; c < p.npad; c += 64) {
    uint32_t v[16];
    tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + c, v);
    tmem_ld_wait();
    if (ok && r < rows) {
      const uint32_t a = smem_u32(part + (size_t)r * pstride + c);
#pragma unroll
      for (int q = 0; q < 4; ++q) st_shared_v4(a + 16 * q, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  }
  if (!ok && threadIdx.x == 0) flag_status(MOE_STATUS_WAIT_TIMEOUT);
  tc_fence_before();
  cluster_sync();  // every CTA's partials are in its shared memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols);

  // ---------------------------------- reduction over the cluster, in order
  const int rpc = (rows + S - 1) / S;
  const int r_lo = min(rows, s * rpc), r_hi = min(rows, r_lo + rpc);
  float* zbuf = reinterpret_cast<float*>(base + L.zbuf);
  const int c4n = p.npad / 4;
  if (S > 1) {
    const uint32_t part_s = smem_u32(part);
    for (int i = threadIdx.x; i < (r_hi - r_lo) * c4n; i += kThreads) {
      const int rr = r_lo + i / c4n, c4 = i % c4n;
      const uint32_t off = part_s + ((uint32_t)rr * pstride + c4 * 4) * 4u;
      // all S remote loads in flight first, then the sum in rank order
      float4 v[kMaxCluster];
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q)
        if (q < S) v[q] = ld_cluster_v4(mapa(off, (uint32_t)q));
      float4 acc = v[0];
#pragma unroll
      for (int q = 1; q < kMaxCluster; ++q)
        if (q < S) {
          acc.x += v[q].x;
          acc.y += v[q].y;
          acc.z += v[q].z;
          acc.w += v[q].w;
        }
      *reinterpret_cast<float4*>(zbuf + (size_t)(rr - r_lo) * p.npad + c4 * 4) = acc;
    }
  }
  __syncthreads();  // this CTA's reduced rows are complete

  // ----------------------------------------------- logits and the top-k
  // (before the exit barrier below: they read only this CTA's own rows, while
  // peers may still be reading its partials)
  auto zrow = [&](int rr) -> const float* {
    return S > 1 ? zbuf + (size_t)(rr - r_lo) * p.npad : part + (size_t)rr * pstride;
  };
  if (p.logits != nullptr)
    for (int i = threadIdx.x; i < (r_hi - r_lo) * p.E; i += kThreads) {
      const int rr = r_lo + i / p.E, e = i % p.E;
      p.logits[(size_t)(row0 + rr) * p.E + e] = zrow(rr)[e];
    }
  if (p.do_topk)
    for (int rr = r_lo + warp; rr < r_hi; rr += kThreads / 32) {
      int e;
      float w;
      bool nan_seen;
      route_token<KEYS>(zrow(rr), p.E, p.k, p.renormalize, lane, e, w, nan_seen);
      const size_t t = (size_t)(row0 + rr);
      if (nan_seen && lane == 0) flag_status(MOE_STATUS_NONFINITE_LOGIT);
      if (lane < p.k) {
        p.topk_idx[t * p.k + lane] = e;
        p.topk_w[t * p.k + lane] = w;
      }
    }
  __syncwarp();
  cluster_sync();  // no CTA leaves while a peer may still read its partials
}

}  // namespace router
}  // namespace moe
