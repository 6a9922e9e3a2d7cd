// grouped_ffn.cuh -- mixed-precision grouped SwiGLU expert FFN for sm_100a.
//
// One persistent launch computes the whole expert FFN: for every expert e and
// every permuted row r of e, the fused gate/up projection with the SwiGLU
// epilogue  h_r = silu(x_r W_g,e^T) * (x_r W_u,e^T)  and then the down
// projection  y_r = h_r W_d,e^T  (ExactMoE, Section 3.4: one fused gate/up
// projection and one down projection per group of experts).  Experts in one
// launch may be BF16, INT8 or INT4 (MxMoE abstract: GEMMs of different
// precisions in one grouped kernel); INT8/INT4 weights are dequantised to bf16
// (q * s exact in fp32, rounded once) in registers inside the mainloop, so no
// bf16 copy of an expert is ever written to global memory (ExactMoE Section
// 3.1: the dequantised values define the operations; no FP16 expert is
// materialised).
//
// Design (one persistent CTA per SM, 16 warps):
//   warp 15      scheduler: takes work units from a global counter -- every
//                gate/up unit, then every down unit, experts in id order with
//                the precisions interleaved -- decodes them and publishes
//                them to the other roles; before publishing a down
//                unit it waits (bounded) until all gate/up epilogues of its
//                expert have published their h rows.
//   warp 0       TMA producer: streams X tiles and BF16 weight boxes into the
//                operand ring (one copy per 128 weight rows).
//   warp 14      code producer: streams INT8/INT4 codes and their fp16 scales
//                into a staging ring, running ahead of the operand stages.
//   warp 1       TMEM owner + MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16
//                -> fp32) into double-buffered TMEM accumulators.
//   warps 2,3,8-13  dequant: staged codes x scale -> bf16, into the shared-
//                memory weight stage (the MMA's B operand in tile mode, its A
//                operand in swap mode).
//   warps 4-7    epilogue: tcgen05.ld, SwiGLU or copy, bf16 stores; gate/up
//                epilogues publish their rows with a release counter.
// A work unit is (projection, expert, block of weight rows, tile of rows of
// that expert).  Weight rows travel in 128-row TMA boxes; a gate/up box holds
// 64 gate rows and the same 64 up rows (a 3-D view of W13), so one epilogue
// sees g and u of the same feature.  Running both projections in one launch
// needs one prologue instead of two, and down units fill the tail of the
// gate/up phase.
//
// Two MMA orientations (the host picks one per launch from T = rows / k):
//   tile mode (large groups, prefill): A = 128 token rows, B = 256 weight rows
//     (two gate/up boxes, or 256 down rows), D = 128 x 256 fp32; TMEM lane =
//     token row.
//   swap mode (small groups, decode): A = 128 weight rows (64 gate + 64 up, or
//     128 down rows), B = the group's rows padded to 16, D = 128 x N; lane =
//     weight row.  The tensor core does no work on padding rows and the small
//     X tiles leave room for a deep weight pipeline, so decode streams weight
//     bytes; the gate/up epilogue exchanges the up half through shared memory.
// CUDA-core units (swap mode): an INT8/INT4 expert with at most fma_rows rows
// (the cold experts of a decode batch, one to a few tokens each) is not run on
// the tensor core, whose rate at such small N is set by the A operand (128 x
// 16 weights per MMA) and falls below the HBM rate of 4-bit weights.  Its units
// flow through the same operand ring -- the producer stages 16 KB of codes, the
// unit's X rows and the group scales per stage, so the ring keeps its full
// depth of bytes in flight -- and the dequant warps compute exact fp32 dot
// products from the codes (f32x2 FMAs); the MMA thread, the epilogue and the
// code producer pass over them.
#pragma once

#include "common.cuh"

namespace moe {
namespace ffn {

constexpr int kThreads = 512;
constexpr int kMaxNS = 12;         // operand stages (64 K-elements each)
constexpr int kMaxNQ = 8;          // staging slots for packed weights
constexpr int kUR = 4;             // work-unit ring depth
constexpr int kMaxE = 512;
constexpr int kBoxRows = 128;      // weight rows per TMA box (gate/up: 64 gate + 64 up)
constexpr int kDequantWarps = 8;   // warps 2, 3, 8 .. 13
constexpr int kDequantThreads = 32 * kDequantWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemLimit = 232448; // dynamic shared memory per block on sm_100
constexpr long long kDrainCycles = 2000000;  // ~1 ms: bound of a wait in the give-up path

// CUDA-core units: token tiles of at most kFmaRows rows; one stage holds 128
// weight rows x 128 code bytes (INT4: 256 K-elements, INT8: 128), then in the
// X part the tile's X rows (kFmaRows x 128 bf16 per 128 K) and the group scales.
constexpr int kFmaRows = 2;
constexpr int kFmaXBytes = 2 * kFmaRows * 256;     // X of an INT4 stage (two 128-K boxes)
constexpr int kFmaScaleBytes = 2 * kBoxRows * 2;   // fp16 scales of two K-groups
constexpr int kFmaMinStages = 16;                  // CUDA-core units only from this K on
constexpr int kFmaXStageMin =                      // X part of a stage, 1024-aligned
    (kFmaXBytes + kFmaScaleBytes + 1023) / 1024 * 1024;

struct alignas(64) ExpertDesc {
  CUtensorMap tm_w13;   // codes/values of [2I][H] as [2][I][H]; box 2 x 64 rows x (64 bf16 | 64 B)
  CUtensorMap tm_w2;    // codes/values of [H][I]; box 128 rows x (64 bf16 | 64 B)
  CUtensorMap tm_q13f;  // INT8/INT4 codes of W13 as [2][I][K bytes]; box 2 x 64 rows x 128 B
  CUtensorMap tm_q2f;   // INT8/INT4 codes of W2; box 128 rows x 128 B
  CUtensorMap tm_s13f;  // INT8/INT4 scales [H/128][2I] as [G][2][I]; box (INT4: 2, INT8: 1) x 2 x 64
  CUtensorMap tm_s2f;   // INT8/INT4 scales [I/128][H]; box (2 | 1) groups x 128 rows
  CUtensorMap tm_q2h;   // INT8/INT4 codes of W2; box 64 rows x 128 B (half-height down units)
  CUtensorMap tm_s2h;   // INT8/INT4 scales [I/128][H]; box (2 | 1) groups x 64 rows
  const __half* s13;    // [H/128][2I]
  const __half* s2;     // [I/128][H]
  int prec;             // MOE_BF16 / MOE_INT8 / MOE_INT4, -1 when unset
  int pad[11];
};
static_assert(sizeof(ExpertDesc) == 1088, "descriptor layout");

struct Unit {
  int e, prec, wrow0, nbox;  // expert, precision, first weight row (of each half), 128-row boxes
  int row0, nrows;           // rows of the token tile
  int flags;                 // kUnitValid | kUnitGateUp | kUnitFma
  int need;                  // gate/up arrivals of the expert (a down unit waits for them)
  int ent;                   // the expert's entry in the unit table
};
constexpr int kUnitValid = 1, kUnitGateUp = 2, kUnitFma = 4;

struct Entry {
  int unit_begin;  // first gate/up unit index of this expert
  int e_prec;      // expert id | precision << 16
  int row0;        // first permuted row of the expert
  int nrows;
};

struct Params {
  const ExpertDesc* descs;
  const int* prec;         // [E] compact copy of descs[e].prec
  const int32_t* offsets;  // [E+1]
  __nv_bfloat16* h;        // [rows][I]: gate/up output, down input
  __nv_bfloat16* y;        // [rows][H]: down output
  int* counter;            // [0] gate/up (swap) or unit (tile) counter, [1] down units
                           // taken (swap), [2] ready slots reserved; zero at launch
  int* done;               // [E] finished gate/up epilogue warps per expert, zero at launch
  int* ready;              // [E] swap mode: entry + 1 of each expert whose gate/up rows are
                           // all published, in that order; zero at launch
  int rows;                // row capacity of x_perm, h and y_perm
  int E, H, I;
  int nwb_gu, nwb_dn;      // weight blocks per expert of each projection
  int xbox_rows;           // rows per X tensor-map box
  int xrows;               // rows of an X stage = rows of a token tile (multiple of 16, <= 128)
  int ns, nq;              // ring depths
  int acc_stride;          // TMEM columns per accumulator buffer
  int fma_rows;            // swap mode: INT8/INT4 experts with <= fma_rows rows run on CUDA cores
};

// Shared-memory map (byte offsets from the 1024-aligned base).
struct SmemMap {
  uint32_t w, x, q, qs, xb, bar, units, misc, entries, total;
  uint32_t wstage, xstage, qslot, qscale;
};

constexpr int kNumBarriers = 96;
// full, empty, wfree, fdone, ffull per stage; qfull, qempty per slot; accfull,
// accempty; ufull, uempty; mmadone, xfull, xempty, go
static_assert(5 * kMaxNS + 2 * kMaxNQ + 2 * 2 + 2 * kUR + 4 <= kNumBarriers, "barrier space");

// ------------------------------------------------------------------- trace --
// Profiling builds only (-DMOE_FFN_TRACE): a per-CTA, per-unit record written
// by every role -- absolute stamps (%globaltimer, ns) and the SM cycles a role
// spent waiting on its barriers for the unit (clock64 sums).  Unit `seq` is the
// CTA's seq-th valid unit; every role receives the units in the same order.
// Read back with moe_ffn_trace_read; the normal build compiles all of it away.
enum TraceField {
  kTrUnit = 0,     // global unit index
  kTrKind,         // flags | prec << 8 | nrows << 16 | expert << 24
  kTrSched,        // ns: scheduler published the unit
  kTrProdBeg,      // ns: producer took the unit
  kTrProdEnd,      // ns: producer issued the unit's last copies
  kTrProdWait,     // cycles: producer waiting on empty
  kTrCodeWait,     // cycles: code producer waiting on qempty
  kTrMmaBeg,       // ns: MMA thread, accumulator buffer free
  kTrMmaEnd,       // ns: MMA thread, last commit issued
  kTrMmaWait,      // cycles: MMA thread waiting on full
  kTrDqBeg,        // ns: dequant warp 2, unit taken (INT8/INT4)
  kTrDqEnd,        // ns: dequant warp 2, last slot handed over
  kTrDqWaitQ,      // cycles: dequant warp 2 waiting on qfull
  kTrDqWaitW,      // cycles: dequant warp 2 waiting on wfree
  kTrEpiBeg,       // ns: epilogue warp 4, accumulator full
  kTrEpiEnd,       // ns: epilogue warp 4, rows stored
  kTrMmaIssue,     // cycles: MMA thread issuing (fence, MMAs, commit)
  kTrDqConv,       // cycles: dequant warp 2 loading and converting codes
  kTrDqStore,      // cycles: dequant warp 2 storing to TMEM and signalling (CUDA-core: output)
  kTrPublish,      // cycles: the gate/up publication (fences + release add)
  kTraceFields
};
#ifdef MOE_FFN_TRACE
constexpr int kTraceCtas = 160, kTraceUnits = 96;
__device__ long long g_ffn_trace[kTraceCtas][kTraceUnits][kTraceFields];
__device__ __forceinline__ void trace_set(int seq, int f, long long v) {
  if (blockIdx.x < kTraceCtas && seq < kTraceUnits) g_ffn_trace[blockIdx.x][seq][f] = v;
}
#define FFN_TRACE_SET(seq, f, v) trace_set((seq), (f), (long long)(v))
#define FFN_TRACE_NS() ((long long)global_timer_ns())
#define FFN_CLOCK() clock64()
#else
#define FFN_TRACE_SET(seq, f, v) ((void)0)
#define FFN_TRACE_NS() 0ll
#define FFN_CLOCK() 0ll
#endif
// Cycle sums are kept in registers during a unit and stored once at its end
// (a global read-modify-write per stage would itself stall the role).

__host__ __device__ inline SmemMap smem_map(bool swap, int ns, int nq, int xrows, int E) {
  SmemMap m;
  const uint32_t wrows = swap ? 128 : 256;
  m.wstage = wrows * 128;
  m.xstage = (uint32_t)xrows * 128;
  if (swap && m.xstage < (uint32_t)kFmaXStageMin) m.xstage = kFmaXStageMin;  // CUDA-core X + scales
  m.qslot = wrows * 64;
  m.qscale = wrows * 2;
  uint32_t off = 0;
  m.w = off;
  off += ns * m.wstage;
  m.x = off;
  off += ns * m.xstage;
  m.q = off;
  off += nq * m.qslot;
  m.qs = off;
  off += nq * m.qscale;
  m.xb = off;
  off += swap ? 64u * xrows * 4u : 0u;
  off = (off + 15) & ~15u;
  m.bar = off;
  off += kNumBarriers * 8;
  m.units = off;
  off += kUR * sizeof(Unit);
  m.misc = off;
  off += 64;
  m.entries = off;
  off += E * sizeof(Entry) + E * sizeof(int);  // entries, then first down unit
  m.total = off + 1024;  // slack to align the dynamic shared-memory base
  return m;
}

struct Smem {
  uint8_t *w_st, *x_st, *q_st, *q_sc;
  float* xbuf;
  uint64_t *full, *empty, *wfree, *qfull, *qempty, *accfull, *accempty, *ufull, *uempty;
  uint64_t *mmadone, *xfull, *xempty, *go, *fdone, *ffull;
  Unit* units;
  uint32_t* tmem_slot;
  int* abort_flag;
  int* n_entries;
  int* n_units;
  int* n_units_gu;
  Entry* entries;
  int* ub_dn;  // [entry] first down unit of the entry's expert
  uint32_t wstage, xstage, qslot, qscale;
};

__device__ __forceinline__ Smem carve(uint8_t* raw, const Params& p, bool swap) {
  const SmemMap m = smem_map(swap, p.ns, p.nq, p.xrows, p.E);
  uint8_t* b = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                          ~uintptr_t(1023));
  Smem s;
  s.w_st = b + m.w;
  s.x_st = b + m.x;
  s.q_st = b + m.q;
  s.q_sc = b + m.qs;
  s.xbuf = reinterpret_cast<float*>(b + m.xb);
  uint64_t* bar = reinterpret_cast<uint64_t*>(b + m.bar);
  s.full = bar;
  s.empty = s.full + kMaxNS;
  s.wfree = s.empty + kMaxNS;
  s.qfull = s.wfree + kMaxNS;
  s.qempty = s.qfull + kMaxNQ;
  s.accfull = s.qempty + kMaxNQ;
  s.accempty = s.accfull + 2;
  s.ufull = s.accempty + 2;
  s.uempty = s.ufull + kUR;
  s.mmadone = s.uempty + kUR;
  s.xfull = s.mmadone + 1;
  s.xempty = s.xfull + 1;
  s.go = s.xempty + 1;
  s.fdone = s.go + 1;
  s.ffull = s.fdone + kMaxNS;
  s.units = reinterpret_cast<Unit*>(b + m.units);
  s.tmem_slot = reinterpret_cast<uint32_t*>(b + m.misc);
  s.abort_flag = reinterpret_cast<int*>(b + m.misc + 4);
  s.n_entries = reinterpret_cast<int*>(b + m.misc + 8);
  s.n_units = reinterpret_cast<int*>(b + m.misc + 12);
  s.n_units_gu = reinterpret_cast<int*>(b + m.misc + 16);
  s.entries = reinterpret_cast<Entry*>(b + m.entries);
  s.ub_dn = reinterpret_cast<int*>(b + m.entries + p.E * sizeof(Entry));
  s.wstage = m.wstage;
  s.xstage = m.xstage;
  s.qslot = m.qslot;
  s.qscale = m.qscale;
  return s;
}

__device__ __forceinline__ void advance(uint32_t& slot, uint32_t& phase, uint32_t n) {
  if (++slot == n) {
    slot = 0;
    phase ^= 1u;
  }
}

#ifdef MOE_FFN_TRACE
// Profiling builds: per CTA, %globaltimer at kernel entry, after the barrier
// and TMEM set-up, after the unit table, at the final barrier and at exit.
__device__ long long g_ffn_kstamp[kTraceCtas][5];
#define FFN_KSTAMP(i)                                                          \
  do {                                                                        \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas)                          \
      g_ffn_kstamp[blockIdx.x][i] = (long long)global_timer_ns();              \
  } while (0)
#else
#define FFN_KSTAMP(i) ((void)0)
#endif

#ifdef MOE_FFN_TRACE
// Profiling builds: the role and unit of the first give-up of each CTA
// ({role, unit sequence number, unit index of that role's last unit}).
__device__ int g_ffn_giveup[kTraceCtas][4];
#endif

// role: 1 scheduler, 2 producer, 3 code producer, 4 MMA, 5 dequant, 6 epilogue
__device__ __forceinline__ void give_up(const Smem& s, int role = 0, int seq = -1) {
#ifdef MOE_FFN_TRACE
  if (blockIdx.x < kTraceCtas && *reinterpret_cast<volatile int*>(s.abort_flag) == 0 &&
      atomicCAS(&g_ffn_giveup[blockIdx.x][0], 0, role) == 0) {
    g_ffn_giveup[blockIdx.x][1] = seq;
    g_ffn_giveup[blockIdx.x][2] = threadIdx.x;
  }
#else
  (void)role;
  (void)seq;
#endif
  *reinterpret_cast<volatile int*>(s.abort_flag) = 1;
  flag_status(MOE_STATUS_WAIT_TIMEOUT);
}

// Token tiles of an expert with n rows (tiles of p.xrows rows, the X stage's
// capacity); each tile is paired with every weight block of a projection.
__device__ __forceinline__ int tiles_of(int n, const Params& p) {
  return n > 0 ? (n + p.xrows - 1) / p.xrows : 0;
}

// CUDA-core down units of an expert (INT8/INT4, at most fma_rows rows, I of at
// least kFmaMinStages stages) are 64 weight rows high, twice as many as the
// 128-row units of the tensor-core path: at one or two tokens per expert a
// down unit streams a long K, and halving it keeps more SMs busy at the end.
template <bool kSwap, bool kFma>
__device__ __forceinline__ bool fma_down(const Params& p, int prec, int nrows) {
  if (!kFma || !kSwap || prec == MOE_BF16 || nrows > p.fma_rows) return false;
  return p.I / (prec == MOE_INT4 ? 256 : 128) >= kFmaMinStages;
}

template <bool kSwap, bool kFma>
__device__ __forceinline__ int down_units_of(const Params& p, int prec, int nrows) {
  return tiles_of(nrows, p) * p.nwb_dn * (fma_down<kSwap, kFma>(p, prec, nrows) ? 2 : 1);
}

// The unit table, built by every CTA from expert_offsets and the precision
// array: the experts with rows, with their first unit index; unit indices =
// every gate/up unit, then every down unit, experts in the same order:
//   swap kernel (decode): ascending id, so precisions are interleaved (hot
//     experts sit at arbitrary ids) and HBM-bound BF16 units run beside the
//     compute-bound CUDA-core units on other SMs (measured faster than putting
//     either kind first); the scheduler hands out gate/up units in this order
//     and down units in the order the experts become ready;
//   tile kernel (prefill): INT4, then INT8, then BF16 experts (ascending id
//     inside a class): the dequant-bound quantised units first, an LPT
//     approximation that leaves the tail to the shorter BF16 units (measured
//     3 % faster there than id order).
// Thread e handles expert e; a block-wide scan (warp shuffles, then the warp
// totals) gives each expert its tile offset and entry index.
// my_prec: p.prec[threadIdx.x] (read by the caller before griddepcontrol.wait:
// the precisions are written only by write_desc_kernel, which never lets a
// dependent launch start before it completes).
template <bool kSwap, bool kFma>
__device__ void build_entries(const Params& p, const Smem& s, int my_prec) {
  static_assert(kThreads >= kMaxE, "one thread per expert");
  constexpr int kWarps = kThreads / 32;
  constexpr int kC = kSwap ? 1 : 3;            // classes in unit order
  int* wsum = reinterpret_cast<int*>(s.q_st);  // [kWarps][3 kC]; staging is free until the mainloop
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int off = 0, n = 0, prec = -1, cls = -1, tiles = 0, dnu = 0;
  if (tid < p.E) {
    off = p.offsets[tid];
    n = p.offsets[tid + 1] - off;
    prec = my_prec;
    // An expert whose rows do not lie inside [0, rows) is left out (no unit
    // reads or writes them) and flagged: the epilogue's stores use these rows.
    if (off < 0 || n < 0 || off > p.rows || n > p.rows - off) {
      if (n != 0) flag_status(MOE_STATUS_BAD_ROW_INDEX);
      n = 0;
    }
    if (n > 0) {
      if (prec == MOE_INT4 || prec == MOE_INT8 || prec == MOE_BF16) {
        cls = kSwap ? 0 : (prec == MOE_INT4 ? 0 : prec == MOE_INT8 ? 1 : 2);
        tiles = tiles_of(n, p);
        dnu = down_units_of<kSwap, kFma>(p, prec, n);
      } else {
        flag_status(MOE_STATUS_UNSET_EXPERT);
      }
    }
  }
  // inclusive warp scans of v[c] = tiles, v[kC + c] = entries and v[2 kC + c]
  // = down units of class c
  int v[3 * kC], incl[3 * kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    v[c] = cls == c ? tiles : 0;
    v[kC + c] = cls == c ? 1 : 0;
    v[2 * kC + c] = cls == c ? dnu : 0;
  }
#pragma unroll
  for (int i = 0; i < 3 * kC; ++i) {
    incl[i] = v[i];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl[i], d);
      if (lane >= d) incl[i] += x;
    }
    if (lane == 31) wsum[warp * 3 * kC + i] = incl[i];
  }
  __syncthreads();
  int before[3 * kC], total[3 * kC];  // sums over earlier warps / over all warps
#pragma unroll
  for (int i = 0; i < 3 * kC; ++i) before[i] = total[i] = 0;
  for (int w = 0; w < kWarps; ++w)
#pragma unroll
    for (int i = 0; i < 3 * kC; ++i) {
      const int x = wsum[w * 3 * kC + i];
      total[i] += x;
      if (w < warp) before[i] += x;
    }
  int total_tiles = 0, total_ents = 0, total_dn = 0;
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    total_tiles += total[c];
    total_ents += total[kC + c];
    total_dn += total[2 * kC + c];
  }
  const int total_gu = total_tiles * p.nwb_gu;
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    if (cls != c) continue;
    int tile_base = 0, ent_base = 0, dn_base = 0;
#pragma unroll
    for (int c2 = 0; c2 < c; ++c2) {
      tile_base += total[c2];
      ent_base += total[kC + c2];
      dn_base += total[2 * kC + c2];
    }
    const int t = tile_base + before[c] + incl[c] - v[c];  // token tiles before this expert
    const int en = ent_base + before[kC + c] + incl[kC + c] - v[kC + c];
    const int dn = dn_base + before[2 * kC + c] + incl[2 * kC + c] - v[2 * kC + c];
    s.entries[en] = Entry{t * p.nwb_gu, tid | (prec << 16), off, n};
    s.ub_dn[en] = total_gu + dn;
  }
  if (tid == 0) {
    *s.n_units_gu = total_gu;
    *s.n_units = total_gu + total_dn;
    *s.n_entries = total_ents;
  }
}

template <bool kSwap, bool kFma>
__device__ __forceinline__ Unit decode_unit(const Params& p, const Smem& s, int u) {
  const bool gu = u < *s.n_units_gu;
  int lo = 0, hi = *s.n_entries - 1;  // last entry whose first unit is <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((gu ? s.entries[mid].unit_begin : s.ub_dn[mid]) <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  const Entry en = s.entries[lo];
  const bool half = !gu && fma_down<kSwap, kFma>(p, en.e_prec >> 16, en.nrows);
  const int nwb = gu ? p.nwb_gu : p.nwb_dn * (half ? 2 : 1);
  const int local = u - (gu ? en.unit_begin : s.ub_dn[lo]);
  const int tt = local / nwb, wb = local % nwb;
  Unit un;
  un.e = en.e_prec & 0xFFFF;
  un.prec = en.e_prec >> 16;
  un.row0 = en.row0 + tt * p.xrows;
  un.nrows = min(p.xrows, en.nrows - tt * p.xrows);
  if (gu) {  // gate rows [wrow0, wrow0 + 64 nbox), up rows I + the same
    un.wrow0 = wb * (kSwap ? 64 : 128);
    un.nbox = kSwap ? 1 : 2;
  } else {
    un.wrow0 = wb * (kSwap ? (half ? kBoxRows / 2 : kBoxRows) : 256);
    un.nbox = half ? 1 : min(kSwap ? 1 : 2, (p.H - un.wrow0) / kBoxRows);
  }
  // CUDA-core units: an INT8/INT4 expert with at most fma_rows rows runs a
  // projection on CUDA cores when its K spans at least kFmaMinStages stages.
  // Shorter units do not repay a unit's fixed costs (first-stage latency, the
  // output stores, the ring stages held while computing): measured on the
  // same B200, gate/up units of K = 2048 (8 INT4 stages) were neutral at the
  // Qwen3-30B-A3B decode shape and 6 % slower at the 512-expert stack shape,
  // while K = 4096 / 14336 (Mixtral-8x7B shape) ran 1.3-1.8x faster.
  const int step = un.prec == MOE_INT4 ? 256 : 128;
  const bool fma_q = kFma && kSwap && un.prec != MOE_BF16 && en.nrows <= p.fma_rows;
  const bool fma_gu = fma_q && p.H / step >= kFmaMinStages;
  const bool fma = gu ? fma_gu : fma_q && p.I / step >= kFmaMinStages;
  un.flags = kUnitValid | (gu ? kUnitGateUp : 0) | (fma ? kUnitFma : 0);
  // gate/up arrivals: the 4 epilogue warps of a tensor-core unit, or every
  // dequant warp of a CUDA-core unit
  un.need = (fma_gu ? kDequantWarps : 4) * tiles_of(en.nrows, p) * p.nwb_gu;
  un.ent = lo;
  return un;
}

__device__ __forceinline__ bool unit_gu(const Unit& un) { return (un.flags & kUnitGateUp) != 0; }

// TMA copy of 128-row box b of a unit's weights (values or codes) at K-column
// kc: gate/up -> gate rows wrow0 + 64 b .. + 63 followed by the same up rows
// (one copy through the [2][I][K] map); down -> rows wrow0 + 128 b .. + 127.
__device__ __forceinline__ void load_weight_box(void* dst, const CUtensorMap* tw, const Unit& un,
                                                int b, int kc, uint64_t* bar) {
  if (un.flags & kUnitGateUp)
    tma_load_3d(dst, tw, kc, un.wrow0 + (kBoxRows / 2) * b, 0, bar);
  else
    tma_load_2d(dst, tw, kc, un.wrow0 + kBoxRows * b, bar);
}

// Bulk copies of the fp16 scales of box b for K-group g, in the box's row
// order (group-major scale arrays: the scales of consecutive rows are
// contiguous).
__device__ __forceinline__ void load_scale_box(void* dst, const Params& p, const ExpertDesc* d,
                                               const Unit& un, int b, int g, uint64_t* bar) {
  if (un.flags & kUnitGateUp) {
    const __half* sc = d->s13 + (size_t)g * (2 * p.I) + un.wrow0 + (kBoxRows / 2) * b;
    constexpr uint32_t kHalfBytes = (kBoxRows / 2) * sizeof(__half);
    bulk_load(dst, sc, kHalfBytes, bar);                                          // gate rows
    bulk_load(static_cast<uint8_t*>(dst) + kHalfBytes, sc + p.I, kHalfBytes, bar);  // up rows
  } else {
    bulk_load(dst, d->s2 + (size_t)g * p.H + un.wrow0 + kBoxRows * b, kBoxRows * sizeof(__half),
              bar);
  }
}

// kFma: the kernel instance has the CUDA-core path.  Without it every CUDA-core
// branch is compiled out: its mere presence (code size, register allocation
// of the roles) cost 7 % of the decode step at shapes that never use it.
template <bool kFma>
__device__ __forceinline__ bool unit_fma(const Unit& un) {
  return kFma && (un.flags & kUnitFma) != 0;
}

// Operand-ring stages of a unit: one per 64-element k-block, or for a CUDA-core
// unit one per 128 code bytes of a row (INT4: 256 K-elements, INT8: 128); the
// last CUDA-core stage may run past K and reads zeros there (TMA fill).
template <bool kFma>
__device__ __forceinline__ int unit_nkb(const Params& p, const Unit& un) {
  const int K = unit_gu(un) ? p.H : p.I;
  if (unit_fma<kFma>(un)) {
    const int step = un.prec == MOE_INT4 ? 256 : 128;
    return (K + step - 1) / step;
  }
  return K / 64;
}

// Bytes a CUDA-core stage receives: codes, X (one or two 128-K boxes) and scales.
// rows: the unit's weight rows (128; 64 for a CUDA-core down unit).
__device__ __forceinline__ uint32_t fma_stage_bytes(int prec, uint32_t rows) {
  const uint32_t boxes = prec == MOE_INT4 ? 2u : 1u;
  return rows * 128 + boxes * (kFmaRows * 256 + rows * 2);
}

__device__ __forceinline__ int ld_acquire(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* ptr, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

__device__ __forceinline__ int atom_release_add(int* ptr, int v) {
  int old;
  asm volatile("atom.release.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void st_release(int* ptr, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Down unit: wait (bounded) until every gate/up epilogue warp of the expert
// has published its h rows.  The acquire makes those writes visible to this
// CTA; the thread that then reads h with TMA orders them before its
// async-proxy reads with fence.proxy.async.global.
__device__ __forceinline__ bool wait_gate_up(const Params& p, const Unit& un,
                                             volatile int* abort_flag) {
  const int* cnt = p.done + un.e;
  const long long t0 = clock64();
  while (ld_acquire(cnt) < un.need) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
    __nanosleep(128);
  }
  return true;
}

// --------------------------------------------------------------- scheduler --
// Takes units from the global counter, decodes them, prefetches the weight
// tensor map and, for a down unit, waits for its gate/up rows, then publishes
// the unit to every role through the unit ring.  It reserves unit n + 1 only
// when the producer reaches the reserve point of unit n (the `go` barrier), a
// few k-blocks before unit n's last copies: every global round trip of a unit
// switch happens here, off the producer's path, while the late reservation
// keeps the dynamic balance of the tail.
template <bool kSwap, bool kFma>
__device__ void scheduler(const Params& p, const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  const int total = *s.n_units;
  uint32_t us = 0, uph = 0, gph = 0;
  int tseq = 0;
  (void)tseq;
  bool ok = true;
  const int total_gu = *s.n_units_gu, total_dn = total - total_gu;
  bool gu_left = true;
  int dn_j = -1, scan_slot = 0, scan_cum = 0;  // swap mode: claimed down unit, ready-list cursor
  const bool uniform_dn = total_dn == *s.n_entries * p.nwb_dn;  // every expert one token tile
  for (bool first = true;; first = false) {
    if (!first) {
      if (!mbar_wait(s.go, gph, abort_flag)) {
        ok = false;
        break;
      }
      gph ^= 1u;
    }
    int u;
    if (!kSwap || !kFma) {
      // every gate/up unit, then every down unit, in order; the first unit of
      // CTA b is unit b, later ones come from the counter.  Without CUDA-core
      // units the gate/up units of an expert finish close together and this
      // order was measured 0.7 % faster at decode than the ready list below.
      u = first ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(p.counter, 1);
    } else if (first && (int)blockIdx.x < total_gu) {
      u = blockIdx.x;
    } else {
      // swap mode: the next gate/up unit (the long units, on the critical
      // path, go first); once none is left, a down unit of an expert whose
      // gate/up rows are all published (experts in the order they became
      // ready), waiting only if no expert is ready.  No SM waits on one expert
      // while another expert's down units are ready.
      // Down unit j (counted in the order the experts became ready) is taken by
      // one atomicAdd, so takers never retry; its expert is found by walking
      // the ready list from this scheduler's cursor (slot, down units before
      // it), waiting only while that slot is not yet filled -- every later
      // slot fills later, so no other down unit could be ready meanwhile.
      u = -1;
      const long long t0 = clock64();
      while (u < 0) {
        if (gu_left) {
          const int g = (int)gridDim.x + atomicAdd(p.counter, 1);
          if (g < total_gu) {
            u = g;
            break;
          }
          gu_left = false;
        }
        if (dn_j < 0) dn_j = atomicAdd(p.counter + 1, 1);
        if (dn_j >= total_dn) {  // every down unit is taken: no work left
          u = total;
          break;
        }
        if (uniform_dn) {  // one token tile per expert: slot = j / (down units per expert)
          const int v = ld_acquire(p.ready + dn_j / p.nwb_dn);
          if (v != 0) {
            u = s.ub_dn[v - 1] + dn_j % p.nwb_dn;
            dn_j = -1;
            break;
          }
          if (*abort_flag || clock64() - t0 > kWaitLimitCycles) break;
          __nanosleep(200);
          continue;
        }
        const int v = ld_acquire(p.ready + scan_slot);
        if (v != 0) {
          const int ent = v - 1;
          const int nd = down_units_of<kSwap, kFma>(p, s.entries[ent].e_prec >> 16,
                                                    s.entries[ent].nrows);
          if (dn_j < scan_cum + nd) {
            u = s.ub_dn[ent] + (dn_j - scan_cum);
            dn_j = -1;
            break;
          }
          scan_cum += nd;
          ++scan_slot;
          continue;
        }
        if (*abort_flag || clock64() - t0 > kWaitLimitCycles) break;
        __nanosleep(200);
      }
      if (u < 0) {
        ok = false;
        break;
      }
    }
    Unit un = Unit{0, 0, 0, 0, 0, 0, 0, 0, 0};
    if (u < total) {
      un = decode_unit<kSwap, kFma>(p, s, u);
      const ExpertDesc* d = p.descs + un.e;
      if (unit_fma<kFma>(un))
        prefetch_tmap(unit_gu(un) ? &d->tm_q13f : &d->tm_q2h);
      else
        prefetch_tmap(unit_gu(un) ? &d->tm_w13 : &d->tm_w2);
      if (!unit_gu(un) && !wait_gate_up(p, un, abort_flag)) {
        ok = false;
        break;
      }
    }
    if (!mbar_wait(&s.uempty[us], uph ^ 1u, abort_flag)) {
      ok = false;
      break;
    }
    s.units[us] = un;
    mbar_arrive(&s.ufull[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    FFN_TRACE_SET(tseq, kTrUnit, u);
    FFN_TRACE_SET(tseq, kTrKind,
                  un.flags | un.prec << 8 | un.nrows << 16 | (long long)un.e << 24);
    FFN_TRACE_SET(tseq, kTrSched, FFN_TRACE_NS());
    ++tseq;
  }
  if (!ok) give_up(s, 1, tseq);
}

// ---------------------------------------------------------------- producer --
// Streams, per k-block, the X tile (one copy) and, for BF16 units, the
// weight boxes into the operand ring.
template <bool kSwap, bool kFma>
__device__ void producer(const CUtensorMap* tm_x, const CUtensorMap* tm_h,
                         const CUtensorMap* tm_xf, const CUtensorMap* tm_hf, const Params& p,
                         const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  const uint32_t ns = p.ns;
  uint32_t st = 0, sph = 0, us = 0, uph = 0;
  // drain bookkeeping: stages with copies issued, whether the last issue was a
  // CUDA-core one (landing on ffull) and the parity of the phase it completes;
  // full and ffull each count phases only at their own kind of position
  uint32_t issued = 0, issued_par = 0, issued_fma = 0, tc_par = 0, fma_par = 0;
  const uint32_t xbytes = (uint32_t)p.xbox_rows * 128;
  bool ok = true;
  int tseq = 0;
  (void)tseq;
  prefetch_tmap(tm_x);
  prefetch_tmap(tm_h);
  if (kSwap) {
    prefetch_tmap(tm_xf);
    prefetch_tmap(tm_hf);
  }
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    FFN_TRACE_SET(tseq, kTrProdBeg, FFN_TRACE_NS());

    const bool gu = unit_gu(un);
    const bool fma = kSwap && unit_fma<kFma>(un);
    const bool int4 = un.prec == MOE_INT4;
    const ExpertDesc* d = p.descs + un.e;
    // (CUDA-core down units are 64 rows high: the half-height maps)
    const CUtensorMap* tw = fma ? (gu ? &d->tm_q13f : &d->tm_q2h) : (gu ? &d->tm_w13 : &d->tm_w2);
    const CUtensorMap* tsc = gu ? &d->tm_s13f : &d->tm_s2h;
    const CUtensorMap* tx = fma ? (gu ? tm_xf : tm_hf) : (gu ? tm_x : tm_h);
    const bool bf16 = un.prec == MOE_BF16;
    if (bf16 || fma) tmap_acquire(tw);
    if (fma) tmap_acquire(tsc);
    if (!gu) fence_proxy_async_global();  // h rows published (scheduler's acquire) -> TMA reads
    const int nkb = unit_nkb<kFma>(p, un);
    const uint32_t bytes = fma ? fma_stage_bytes(un.prec, gu ? kBoxRows : kBoxRows / 2)
                               : xbytes + (bf16 ? (uint32_t)un.nbox * (kBoxRows * 128) : 0u);
    const int reserve_kb = max(0, nkb - (int)ns - 4);
    long long tr_wait = 0;
    (void)tr_wait;
    for (int kb = 0; kb < nkb; ++kb) {
      if (kb == reserve_kb) mbar_arrive(s.go);
      const long long c0 = FFN_CLOCK();
      bool freed;
      if (kFma) {
        // The stage's last use decides what frees it: the MMA commit on empty
        // after a tensor-core position, all dequant warps' arrivals on fdone
        // after a CUDA-core one.  Each barrier completes once per use of its
        // kind, so the parity is that of the use-count bit (tc_par / fma_par).
        const uint32_t bit = 1u << st;
        if (!(issued & bit))
          freed = true;  // never filled
        else if (issued_fma & bit)
          freed = mbar_wait(&s.fdone[st], ((fma_par >> st) & 1u) ^ 1u, abort_flag);
        else
          freed = mbar_wait(&s.empty[st], ((tc_par >> st) & 1u) ^ 1u, abort_flag);
      } else {
        freed = mbar_wait(&s.empty[st], sph ^ 1u, abort_flag);
      }
      if (!freed) {
        ok = false;
        break;
      }
      tr_wait += FFN_CLOCK() - c0;
      if (fma) {
        // CUDA-core position: the data lands on ffull[st], which completes only
        // at such positions, so the dequant warps count its phases per stage no
        // matter how many tensor-core positions lie in between (and the MMA
        // thread, which passes over these positions, counts full's likewise).
        mbar_arrive_expect_tx(&s.ffull[st], bytes);
        // 128 code bytes of each of the 128 weight rows, the tile's X rows for
        // the same K range (one or two 128-element boxes) and the K-groups'
        // scales; the dequant warps compute the stage on CUDA cores.
        uint8_t* xdst = s.x_st + st * s.xstage;
        uint64_t* fb = &s.ffull[st];
        const int k0 = kb * (int4 ? 256 : 128), g0 = kb * (int4 ? 2 : 1);
        if (gu)
          tma_load_3d(s.w_st + st * s.wstage, tw, kb * 128, un.wrow0, 0, fb);
        else
          tma_load_2d(s.w_st + st * s.wstage, tw, kb * 128, un.wrow0, fb);
        tma_load_2d(xdst, tx, k0, un.row0, fb);
        if (int4) tma_load_2d(xdst + kFmaRows * 256, tx, k0 + 128, un.row0, fb);
        if (gu)
          tma_load_3d(xdst + kFmaXBytes, tsc, un.wrow0, 0, g0, fb);
        else
          tma_load_2d(xdst + kFmaXBytes, tsc, un.wrow0, g0, fb);
        issued_fma |= 1u << st;
        issued_par = (issued_par & ~(1u << st)) | (((fma_par >> st) & 1u) << st);
        fma_par ^= 1u << st;
      } else {
        // INT8/INT4 tensor-core position: the dequant warps may fill this
        // stage.  They pass over BF16 units without waiting and may be ring
        // revolutions ahead; wfree, complete only at these positions, tells
        // them the producer has reached it.
        if (!bf16) mbar_arrive(&s.wfree[st]);
        mbar_arrive_expect_tx(&s.full[st], bytes);
        if (bf16) mbar_arrive_n(&s.full[st], kDequantWarps);  // no dequant at this position
        tma_load_2d(s.x_st + st * s.xstage, tx, kb * 64, un.row0, &s.full[st]);
        if (bf16)
          for (int b = 0; b < un.nbox; ++b)
            load_weight_box(s.w_st + st * s.wstage + b * (kBoxRows * 128), tw, un, b, kb * 64,
                            &s.full[st]);
        issued_fma &= ~(1u << st);
        issued_par = (issued_par & ~(1u << st)) | (((tc_par >> st) & 1u) << st);
        tc_par ^= 1u << st;
      }
      issued |= 1u << st;
      advance(st, sph, ns);
    }
    if (!ok) break;
    FFN_TRACE_SET(tseq, kTrProdEnd, FFN_TRACE_NS());
    FFN_TRACE_SET(tseq, kTrProdWait, tr_wait);
    ++tseq;
  }
  if (!ok) {
    give_up(s, 2, tseq);
    // Let copies already in flight land before the CTA's shared memory goes
    // away.  The full barrier of an INT8/INT4 position also counts dequant
    // arrivals, which may never come once the CTA gives up, so each wait is
    // cut short after about a millisecond (copies land within microseconds).
    for (uint32_t i = 0; i < ns; ++i)
      if (issued & (1u << i))
        mbar_wait((issued_fma >> i) & 1u ? &s.ffull[i] : &s.full[i], (issued_par >> i) & 1u,
                  nullptr, kDrainCycles);
  }
}

// ------------------------------------------------------------ code producer --
// Streams the INT8/INT4 codes and fp16 scales of each quantised unit into the
// staging ring, as far ahead as the ring allows, independently of the operand
// stages (which wait on the tensor core); BF16 units are skipped.
template <bool kFma>
__device__ void code_producer(const Params& p, const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  const uint32_t nq = p.nq;
  uint32_t q = 0, qph = 0, us = 0, uph = 0;
  uint32_t qissued = 0, qissued_par = 0;  // drain bookkeeping
  bool ok = true;
  int tseq = -1;
  (void)tseq;
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    ++tseq;
    if (un.prec == MOE_BF16 || unit_fma<kFma>(un)) continue;
    const bool gu = unit_gu(un);
    const ExpertDesc* d = p.descs + un.e;
    const CUtensorMap* tw = gu ? &d->tm_w13 : &d->tm_w2;
    tmap_acquire(tw);
    prefetch_tmap(tw);
    const int nkb = unit_nkb<kFma>(p, un);
    const bool int4 = un.prec == MOE_INT4;
    long long tr_wait = 0;
    (void)tr_wait;
    for (int kb = 0; kb < nkb; kb += int4 ? 2 : 1) {
      const long long c0 = FFN_CLOCK();
      if (!mbar_wait(&s.qempty[q], qph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      tr_wait += FFN_CLOCK() - c0;
      mbar_arrive_expect_tx(&s.qfull[q], (uint32_t)un.nbox * (kBoxRows * 64 + kBoxRows * 2));
      const int kc = int4 ? (kb >> 1) * 64 : kb * 64;  // byte column of the codes
      const int g = kb >> 1;                            // K-group of the scales
      for (int b = 0; b < un.nbox; ++b) {
        load_weight_box(s.q_st + q * s.qslot + b * (kBoxRows * 64), tw, un, b, kc, &s.qfull[q]);
        load_scale_box(s.q_sc + q * s.qscale + b * (kBoxRows * 2), p, d, un, b, g, &s.qfull[q]);
      }
      qissued |= 1u << q;
      qissued_par = (qissued_par & ~(1u << q)) | (qph << q);
      advance(q, qph, nq);
    }
    if (!ok) break;
    FFN_TRACE_SET(tseq, kTrCodeWait, tr_wait);
  }
  if (!ok) {
    give_up(s, 3, tseq);
    for (uint32_t i = 0; i < nq; ++i)
      if (qissued & (1u << i)) mbar_wait(&s.qfull[i], (qissued_par >> i) & 1u);
  }
}

// -------------------------------------------------------------- MMA issuer --
// TMEM columns: tile mode uses two 256-column accumulators; swap mode uses two
// accumulators of acc_stride columns (the power of two >= the token tile, so
// N <= acc_stride).  Every MMA reads both operands from shared memory: in swap
// mode the dequantised INT8/INT4 weights are written into the weight stage in
// the layout a BF16 box arrives in (measured 1 % faster for the decode FFN
// than A operands in TMEM, whose MMA form issued ~1.5x slower per stage).

// Four K=16 MMAs over one 64-element k-block.  The operand descriptors are
// formed once per stage by adding to base descriptors (the start-address field
// is the low 14 bits, in 16-byte units; +2 per 32-byte K step inside the
// 128-byte swizzle row), and the sequence is fully unrolled with no branch
// between the MMAs: in this form the issuing thread keeps the tensor core fed
// (about 4x cheaper per MMA than computing each descriptor in the loop).
__device__ __forceinline__ void mma_kblock_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t acc0) {
  mma_bf16_ss(d, a, b, idesc, acc0);
  mma_bf16_ss(d, a + 2, b + 2, idesc, 1u);
  mma_bf16_ss(d, a + 4, b + 4, idesc, 1u);
  mma_bf16_ss(d, a + 6, b + 6, idesc, 1u);
}

template <bool kSwap, bool kFma>
__device__ void mma_issuer(const Params& p, const Smem& s, uint32_t tmem) {
  const uint32_t acc_cols = p.acc_stride;
  volatile int* abort_flag = s.abort_flag;
  const uint32_t ns = p.ns;
  const uint64_t wdesc0 = smem_desc_sw128(smem_u32(s.w_st));
  const uint64_t xdesc0 = smem_desc_sw128(smem_u32(s.x_st));
  const uint32_t wstep = s.wstage >> 4, xstep = s.xstage >> 4;
  uint32_t st = 0, sph = 0, us = 0, uph = 0, abuf = 0;
  uint32_t tph = 0;  // full phase bit per stage: it only advances at tensor-core positions
  uint32_t aph[2] = {0, 0};
  bool ok = true;
  int tseq = 0;
  (void)tseq;
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    const int nkb = unit_nkb<kFma>(p, un);
    if (kSwap && unit_fma<kFma>(un)) {  // computed and freed by the dequant warps
      for (int kb = 0; kb < nkb; ++kb) advance(st, sph, ns);
      ++tseq;
      continue;
    }
    if (!mbar_wait(&s.accempty[abuf], aph[abuf] ^ 1u, abort_flag)) {
      ok = false;
      break;
    }
    tc_fence_after();
    FFN_TRACE_SET(tseq, kTrMmaBeg, FFN_TRACE_NS());
    const uint32_t d_tmem = tmem + abuf * acc_cols;
    const int n = kSwap ? max(16, (un.nrows + 15) & ~15) : un.nbox * kBoxRows;
    const uint32_t idesc = idesc_bf16_f32(128, n);
    long long tr_wait = 0, tr_issue = 0;
    (void)tr_wait;
    (void)tr_issue;
    for (int kb = 0; kb < nkb; ++kb) {
      const long long c0 = FFN_CLOCK();
      if (!mbar_wait(&s.full[st], (tph >> st) & 1u, abort_flag)) {  // X landed, weights in place
        ok = false;
        break;
      }
      tph ^= 1u << st;
      const long long c1 = FFN_CLOCK();
      tr_wait += c1 - c0;
      tc_fence_after();
      const uint64_t xd = xdesc0 + st * xstep, wd = wdesc0 + st * wstep;
      const uint32_t acc0 = kb != 0;
      if (kSwap)
        mma_kblock_ss(d_tmem, wd, xd, idesc, acc0);
      else
        mma_kblock_ss(d_tmem, xd, wd, idesc, acc0);
      mma_commit(&s.empty[st]);
      advance(st, sph, ns);
      tr_issue += FFN_CLOCK() - c1;
    }
    if (!ok) break;
    mma_commit(&s.accfull[abuf]);
    FFN_TRACE_SET(tseq, kTrMmaEnd, FFN_TRACE_NS());
    FFN_TRACE_SET(tseq, kTrMmaWait, tr_wait);
    FFN_TRACE_SET(tseq, kTrMmaIssue, tr_issue);
    ++tseq;
    aph[abuf] ^= 1u;
    abuf ^= 1u;
  }
  if (!ok) give_up(s, 4, tseq);
  // All issued MMAs must finish before TMEM is released.
  mma_commit(s.mmadone);
  mbar_wait(s.mmadone, 0);
}

// ----------------------------------------------------------------- dequant --
// The dequant warps take part only in INT8/INT4 positions of the operand ring
// and pass over BF16 units at once, so they may be any number of ring
// revolutions away from the producer and the MMA; a parity wait on a barrier
// that completes at every position (empty) could then match the wrong phase.
// They wait instead on wfree[st], which the producer arrives on (after its own
// empty wait, i.e. once the previous use of the stage is complete) only at
// INT8/INT4 positions, and count its phases per stage: at most one phase of
// wfree[st] is ever outstanding, so the parity is exact.


// Code -> bf16 dequantisation, exact up to the final rounding.  A code byte u
// (INT4: the nibble, u = q + 8; INT8: the byte xor 0x80, u = q + 128) becomes
// the fp32 m = 2^15 + u by placing it in mantissa bits 8..15 of 2^15 (one
// prmt).  Then fma(m, s, -(2^15 + off) * s) = (u - off) * s = q * s, where the
// constant is exact in fp32 ((2^15 + 8) * s needs 24 bits, (2^15 + 128) * s
// 20 bits, s being fp16) and the fused product-sum is rounded once, so the
// fp32 result is q * s exactly; cvt.rn.bf16x2 then rounds it to bf16.
__device__ __forceinline__ uint32_t place_byte(uint32_t src, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0x47000000, %2;" : "=r"(d) : "r"(src), "r"(sel));
  return d;
}

// Two codes (byte b0 of src0, byte b1 of src1) -> packed bf16x2 of q * s.
__device__ __forceinline__ uint32_t deq2(uint32_t src0, uint32_t sel0, uint32_t src1,
                                         uint32_t sel1, uint64_t s2, uint64_t c2) {
  uint64_t m, w;
  asm("mov.b64 %0, {%1, %2};" : "=l"(m) : "r"(place_byte(src0, sel0)), "r"(place_byte(src1, sel1)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(w) : "l"(m), "l"(s2), "l"(c2));
  uint32_t lo, hi, d;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(w));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "r"(hi), "r"(lo));
  return d;
}

// prmt selector that puts byte b of the first operand into bits 8..15 over
// 0x47000000 (bytes 0 and 2 zero, byte 3 = 0x47).
__device__ __forceinline__ constexpr uint32_t sel_byte(uint32_t b) { return 0x7604u | (b << 4); }

__device__ __forceinline__ uint64_t f32x2(float v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// Gate/up results: once this warp's h stores are done, publish them to the
// down units of the expert (release counter; the proxy fence orders the
// generic-proxy stores before any TMA read that the counter enables).
// Ordering: each lane's proxy fence orders its generic-proxy h stores for the
// async proxy (the TMA reads of the down units); __syncwarp orders the lanes'
// stores before lane 0's release add, whose gpu-scope release covers them
// (cumulativity), so no full fence is needed.  The arrival that completes the
// expert's count appends the expert's entry to the ready list (swap mode's
// scheduler takes down units from it): its atomic add reads every earlier
// release on the counter, and the release store of the list entry carries
// them on to the scheduler's acquire.
__device__ __forceinline__ void publish_rows(const Params& p, const Unit& un, int lane) {
  fence_proxy_async_global();
  __syncwarp();
  if (lane == 0) {
    const int old = atom_release_add(p.done + un.e, 1);
    if (old + 1 == un.need) st_release(p.ready + atomicAdd(p.counter + 2, 1), un.ent + 1);
  }
}

// ------------------------------------------------------- CUDA-core units --
// A stage holds 128 weight rows x 128 code bytes ([2][64][128] for gate/up:
// gate rows, then the same up rows), X as [box][kFmaRows][128] bf16 and the
// scales as [group][128 rows] fp16.  Dequant thread ft (0..255) owns K-chunk
// c = ft % 16 of every row 16 j + ft / 16 (j = 0..7): 8 code bytes, i.e. 16
// INT4 or 8 INT8 elements; a warp's code loads cover 256 contiguous bytes.  Its
// X values (fp32 pairs) are loaded once per stage and serve all 8 rows.  Rows
// j and j + 4 of a gate/up unit are a gate row and its up row, so the SwiGLU
// needs no exchange.  Dot products are exact-product fp32 sums:
//   INT4: a code u becomes the fp32 value 128 + u (u placed in bits 16..19 of
//     128.0, one prmt); sum_k (128 + u_k) x_k - 136 sum_k x_k = sum_k q_k x_k
//     with q = u - 8, every product exact (8 x 8 significant bits);
//   INT8: 32768 + (q + 128) (the byte in bits 8..15 of 2^15), minus 32896
//     exactly, then exact products.
// The K-group's scale multiplies each partial sum (fp32), the 16 lanes of a
// row are summed at the end of the unit, and the results are rounded to bf16
// once (h = silu(g) * u for gate/up, y for down).

__device__ __forceinline__ uint64_t pack_f32x2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ float hsum2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return __uint_as_float(lo) + __uint_as_float(hi);
}

// bf16x2 word (element 2i in the low half) -> fp32 pair, exactly.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return pack_f32x2(w << 16, w & 0xFFFF0000u);
}

// Byte b of a (an INT4 nibble 0..15) -> fp32 128 + nibble.
__device__ __forceinline__ uint32_t nib_f32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0x43000000, %2;" : "=r"(d) : "r"(a), "r"(0x7044u | (b << 8)));
  return d;
}

template <int N, bool kInt4, bool kHalf>
__device__ __forceinline__ bool fma_unit(const Params& p, const Smem& s, const Unit& un, int ft,
                                         uint32_t& st, uint32_t& sph, uint32_t& ffph, Unit& pub,
                                         long long* tr) {
  long long& tr_wait = tr[0];
  long long& tr_conv = tr[1];
  long long& tr_out = tr[3];
  long long& tr_pub = tr[4];
  (void)tr_out;
  (void)tr_pub;
  volatile int* abort_flag = s.abort_flag;
  const uint32_t ns = p.ns;
  const int lane = threadIdx.x & 31;
  const int c = ft & 15, rsub = ft >> 4;
  constexpr int kPairs = kInt4 ? 8 : 4;  // element pairs of a lane's chunk
  const int nkb = unit_nkb<true>(p, un);
  constexpr int kJ = kHalf ? 4 : 8;  // rows 16 j + rsub of the unit (128, or 64 for kHalf)
  float acc[8][N];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int n = 0; n < N; ++n) acc[j][n] = 0.0f;
  const uint64_t off2 = pack_f32x2(__float_as_uint(-32896.0f), __float_as_uint(-32896.0f));
  const uint64_t one2 = pack_f32x2(__float_as_uint(1.0f), __float_as_uint(1.0f));
  (void)off2;
  (void)one2;
  for (int kb = 0; kb < nkb; ++kb) {
    // ffull counts phases at CUDA-core positions only (bits in ffph, per stage)
    const long long c0 = FFN_CLOCK();
    if (!mbar_wait(&s.ffull[st], (ffph >> st) & 1u, abort_flag)) return false;
    ffph ^= 1u << st;
    const long long c1 = FFN_CLOCK();
    tr_wait += c1 - c0;
    const uint8_t* xs = s.x_st + st * s.xstage;
    const uint8_t* codes = s.w_st + st * s.wstage;
    // X of this lane's chunk, fp32 pairs, and (INT4) its per-token sum
    uint64_t xv[N][kPairs];
    float sx[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
      if (kInt4) {
        const uint4* src = reinterpret_cast<const uint4*>(xs + (c >> 3) * (kFmaRows * 256) +
                                                          n * 256 + (c & 7) * 32);
        const uint4 a = src[0], b = src[1];
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float t = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xv[n][i] = bf16x2_to_f32x2(w[i]);
          t += hsum2(xv[n][i]);
        }
        sx[n] = t;
      } else {
        const uint4 a = *reinterpret_cast<const uint4*>(xs + n * 256 + c * 16);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[n][i % kPairs] = bf16x2_to_f32x2(w[i]);
        sx[n] = 0.0f;
      }
    }
    const __half* sc = reinterpret_cast<const __half*>(xs + kFmaXBytes) +
                       (kInt4 ? (c >> 3) * (kHalf ? kBoxRows / 2 : kBoxRows) : 0);
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
      const int r = 16 * j + rsub;
      const uint2 w = *reinterpret_cast<const uint2*>(codes + r * 128 + c * 8);
      const float sr = __half2float(sc[r]);
      uint64_t d[N];
#pragma unroll
      for (int n = 0; n < N; ++n) d[n] = 0;
      if (kInt4) {
        const uint32_t wd[2] = {w.x, w.y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t lo = wd[h] & 0x0F0F0F0Fu, hi = (wd[h] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint64_t m = pack_f32x2(nib_f32(lo, b), nib_f32(hi, b));  // elements 2i, 2i+1
#pragma unroll
            for (int n = 0; n < N; ++n) d[n] = ffma2(m, xv[n][4 * h + b], d[n]);
          }
        }
#pragma unroll
        for (int n = 0; n < N; ++n)
          acc[j][n] = fmaf(sr, fmaf(-136.0f, sx[n], hsum2(d[n])), acc[j][n]);
      } else {
        const uint32_t wd[2] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint64_t m = pack_f32x2(place_byte(wd[h], sel_byte(2 * b)),
                                          place_byte(wd[h], sel_byte(2 * b + 1)));
            const uint64_t q = ffma2(m, one2, off2);  // exact: the integer q of each code
#pragma unroll
            for (int n = 0; n < N; ++n) d[n] = ffma2(q, xv[n][(2 * h + b) % kPairs], d[n]);
          }
#pragma unroll
        for (int n = 0; n < N; ++n) acc[j][n] = fmaf(sr, hsum2(d[n]), acc[j][n]);
      }
    }
    tr_conv += FFN_CLOCK() - c1;
    // This warp is done with the stage; the producer refills it once all
    // eight dequant warps have arrived (no warp waits for the others).
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.fdone[st]);
    advance(st, sph, ns);
    // the previous gate/up unit's h rows, stored a stage ago: publishing them
    // now costs little (the fence no longer waits for stores in flight)
    if (pub.flags & kUnitValid) {
      publish_rows(p, pub, lane);
      pub.flags = 0;
    }
  }
  const long long c3 = FFN_CLOCK();
  // sum the 16 lanes (K-chunks) of each row; every lane ends with the totals
#pragma unroll
  for (int j = 0; j < kJ; ++j)
#pragma unroll
    for (int n = 0; n < N; ++n) {
      float v = acc[j][n];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      acc[j][n] = v;
    }
  if (unit_gu(un)) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int n = 0; n < N; ++n)
        if (c == n && n < un.nrows)
          p.h[(size_t)(un.row0 + n) * p.I + un.wrow0 + 16 * j + rsub] =
              __float2bfloat16_rn(silu_mul(acc[j][n], acc[j + 4][n]));
    pub = un;  // published later (deferred publication)
  } else {
#pragma unroll
    for (int j = 0; j < kJ; ++j)
#pragma unroll
      for (int n = 0; n < N; ++n)
        if (c == n && n < un.nrows)
          p.y[(size_t)(un.row0 + n) * p.H + un.wrow0 + 16 * j + rsub] =
              __float2bfloat16_rn(acc[j][n]);
  }
  tr_out += FFN_CLOCK() - c3;
  return true;
}

template <bool kInt4>
__device__ bool fma_dispatch(const Params& p, const Smem& s, const Unit& un, int ft, uint32_t& st,
                             uint32_t& sph, uint32_t& ffph, Unit& pub, long long* tr) {
  static_assert(kFmaRows >= 1 && kFmaRows <= 2, "CUDA-core tiles of 1 or 2 rows");
  if (!unit_gu(un)) {  // down units: 64 weight rows
    if (kFmaRows >= 2 && un.nrows == 2)
      return fma_unit<2, kInt4, true>(p, s, un, ft, st, sph, ffph, pub, tr);
    return fma_unit<1, kInt4, true>(p, s, un, ft, st, sph, ffph, pub, tr);
  }
  if (kFmaRows >= 2 && un.nrows == 2)
    return fma_unit<2, kInt4, false>(p, s, un, ft, st, sph, ffph, pub, tr);
  return fma_unit<1, kInt4, false>(p, s, un, ft, st, sph, ffph, pub, tr);
}

// One staging slot holds an INT4 group (128 K-elements = two k-blocks) or an
// INT8 k-block (64 K-elements) for the unit's weight rows, 64 bytes per row.
// Work item = 16 bytes of codes of one row: INT4 -> 32 elements (4 output
// chunks of 8), INT8 -> 16 elements (2 chunks).  A thread loads all its items
// first, then converts and stores them in the 128-byte-swizzled K-major layout
// (chunk c of row r at r * 128 + ((c ^ (r & 7)) << 4)).  Each warp signals
// its own part (barrier counts are kDequantWarps), so the warps never wait on
// one another.
// Swap mode: dequantised weights go into the stage's weight buffer, laid out
// as a BF16 box arrives (rows of 128 bytes, 16-byte chunks swizzled by row & 7,
// so the 32 rows of a warp's stores hit distinct banks).  Warp w owns weight
// rows 32 (w % 4) .. + 31 of the unit (one row per thread) and one half of each
// staging slot (warps 10..13 the second half): INT4 slot = two k-blocks (half h
// -> k-block 2g + h, 32 code bytes -> 64 elements -> 8 chunks), INT8 slot = one
// k-block (half h -> elements 32 h .. + 31 -> chunks 4 h .. 4 h + 3).
template <bool kFma>
__device__ void dequant_swap(const Params& p, const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int half = warp >= 10 ? 1 : 0;
  const int r = quarter * 32 + lane;  // weight row of the unit
  const uint32_t ns = p.ns, nq = p.nq;
  uint32_t st = 0, sph = 0, q = 0, qph = 0, us = 0, uph = 0;
  uint32_t fph = 0;   // wfree phase bit per stage: INT8/INT4 tensor-core positions only
  uint32_t ffph = 0;  // ffull phase bit per stage: CUDA-core positions only
  const int ft = (warp < 4 ? warp - 2 : warp - 6) * 32 + lane;  // warps 2, 3, 8 .. 13
  // A CUDA-core gate/up unit's h rows are published (fence + release add) one
  // stage into the next CUDA-core unit, when their stores have landed -- and
  // always before this warp could block on anything a down unit's wait could
  // hold up: the unit ring, or an INT8/INT4 tensor-core unit.
  Unit pub = Unit{0, 0, 0, 0, 0, 0, 0, 0, 0};  // flags != 0: a publication is pending
  bool ok = true;
  int tseq = -1;
  const bool tracer = warp == 2 && lane == 0;
  (void)tseq;
  (void)tracer;
  for (;;) {
    if ((pub.flags & kUnitValid) && !mbar_try_wait(&s.ufull[us], uph)) {
      publish_rows(p, pub, lane);
      pub.flags = 0;
    }
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    ++tseq;
    const int nkb = unit_nkb<kFma>(p, un);
    if ((pub.flags & kUnitValid) && !unit_fma<kFma>(un)) {
      publish_rows(p, pub, lane);
      pub.flags = 0;
    }
    if (un.prec == MOE_BF16) {
      for (int kb = 0; kb < nkb; ++kb) advance(st, sph, ns);
      continue;
    }
    if (tracer) FFN_TRACE_SET(tseq, kTrDqBeg, FFN_TRACE_NS());
    if (unit_fma<kFma>(un)) {
      long long tr[5] = {0, 0, 0, 0, 0};
      ok = un.prec == MOE_INT4
               ? fma_dispatch<true>(p, s, un, ft, st, sph, ffph, pub, tr)
               : fma_dispatch<false>(p, s, un, ft, st, sph, ffph, pub, tr);
      if (!ok) break;
      if (tracer) {
        FFN_TRACE_SET(tseq, kTrDqEnd, FFN_TRACE_NS());
        FFN_TRACE_SET(tseq, kTrDqWaitQ, tr[0]);
        FFN_TRACE_SET(tseq, kTrDqConv, tr[1]);
        FFN_TRACE_SET(tseq, kTrDqWaitW, tr[2]);
        FFN_TRACE_SET(tseq, kTrDqStore, tr[3]);
        FFN_TRACE_SET(tseq, kTrPublish, tr[4]);
      }
      continue;
    }
    const bool int4 = un.prec == MOE_INT4;
    const float off = int4 ? 32776.0f : 32896.0f;  // 2^15 + 8, 2^15 + 128
    long long tr_wq = 0, tr_ww = 0, tr_conv = 0, tr_store = 0;
    (void)tr_wq;
    (void)tr_ww;
    (void)tr_conv;
    (void)tr_store;
    for (int kb = 0; kb < nkb; kb += int4 ? 2 : 1) {
      const uint32_t st0 = st;
      advance(st, sph, ns);
      const uint32_t st1 = st;
      if (int4) advance(st, sph, ns);
      const long long tq0 = FFN_CLOCK();
      if (!mbar_wait(&s.qfull[q], qph, abort_flag)) {
        ok = false;
        break;
      }
      const long long tq1 = FFN_CLOCK();
      if (!mbar_wait(&s.wfree[st0], (fph >> st0) & 1u, abort_flag) ||
          (int4 && !mbar_wait(&s.wfree[st1], (fph >> st1) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      const long long tq2 = FFN_CLOCK();
      tr_wq += tq1 - tq0;
      tr_ww += tq2 - tq1;
      fph ^= (1u << st0) | (int4 ? 1u << st1 : 0u);
      const uint4* src = reinterpret_cast<const uint4*>(s.q_st + q * s.qslot + r * 64 + half * 32);
      const uint4 c0 = src[0], c1 = src[1];
      const float sc = __half2float(reinterpret_cast<const __half*>(s.q_sc + q * s.qscale)[r]);
      const uint64_t s2 = f32x2(sc), k2 = f32x2(-off * sc);
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      if (int4) {
        uint32_t v[32];  // word j = elements 8 j .. 8 j + 7 -> columns 4 j .. 4 j + 3
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t lo = w[j] & 0x0F0F0F0Fu, hi = (w[j] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int b = 0; b < 4; ++b) v[4 * j + b] = deq2(lo, sel_byte(b), hi, sel_byte(b), s2, k2);
        }
        tr_conv += FFN_CLOCK() - tq2;
        const uint32_t row = smem_u32(s.w_st + (half ? st1 : st0) * s.wstage) + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(row + ((c ^ (r & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2],
                       v[4 * c + 3]);
      } else {
        uint32_t v[16];  // word j = elements 4 j .. 4 j + 3 -> columns 2 j, 2 j + 1
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t a = w[j] ^ 0x80808080u;
          v[2 * j] = deq2(a, sel_byte(0), a, sel_byte(1), s2, k2);
          v[2 * j + 1] = deq2(a, sel_byte(2), a, sel_byte(3), s2, k2);
        }
        tr_conv += FFN_CLOCK() - tq2;
        const uint32_t row = smem_u32(s.w_st + st0 * s.wstage) + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int cc = half * 4 + c;
          st_shared_v4(row + ((cc ^ (r & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2],
                       v[4 * c + 3]);
        }
      }
      const long long tq3 = FFN_CLOCK();
      fence_proxy_async_smem();  // the tensor core (async proxy) reads these bytes
      __syncwarp();
      if (lane == 0) {  // one arrival per dequant warp and stage
        mbar_arrive(&s.full[st0]);
        if (int4) mbar_arrive(&s.full[st1]);
        mbar_arrive(&s.qempty[q]);
      }
      advance(q, qph, nq);
      tr_store += FFN_CLOCK() - tq3;
    }
    if (!ok) break;
    if (tracer) {
      FFN_TRACE_SET(tseq, kTrDqEnd, FFN_TRACE_NS());
      FFN_TRACE_SET(tseq, kTrDqWaitQ, tr_wq);
      FFN_TRACE_SET(tseq, kTrDqWaitW, tr_ww);
      FFN_TRACE_SET(tseq, kTrDqConv, tr_conv);
      FFN_TRACE_SET(tseq, kTrDqStore, tr_store);
    }
  }
  if (pub.flags & kUnitValid) publish_rows(p, pub, lane);
  if (!ok) give_up(s, 5, tseq);
}

__device__ void dequant(const Params& p, const Smem& s, int dtid) {
  volatile int* abort_flag = s.abort_flag;
  const int lane = threadIdx.x & 31;
  const uint32_t ns = p.ns, nq = p.nq;
  uint32_t st = 0, sph = 0, q = 0, qph = 0, us = 0, uph = 0;
  uint32_t fph = 0;  // wfree phase bit per stage: it only advances on INT8/INT4 positions
  constexpr int kMaxItems = 4;  // 256 rows x 4 items / kDequantThreads
  bool ok = true;
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    const int nkb = unit_nkb<false>(p, un);
    if (un.prec == MOE_BF16) {
      for (int kb = 0; kb < nkb; ++kb) advance(st, sph, ns);
      continue;
    }
    const bool int4 = un.prec == MOE_INT4;
    const int items = un.nbox * kBoxRows * 4;
    const float off = int4 ? 32776.0f : 32896.0f;  // 2^15 + 8, 2^15 + 128
    const uint32_t flip = int4 ? 0u : 0x80808080u;
    for (int kb = 0; kb < nkb; kb += int4 ? 2 : 1) {
      const uint32_t st0 = st;
      advance(st, sph, ns);
      const uint32_t st1 = st;
      if (int4) advance(st, sph, ns);
      if (!mbar_wait(&s.qfull[q], qph, abort_flag) ||
          !mbar_wait(&s.wfree[st0], (fph >> st0) & 1u, abort_flag) ||
          (int4 && !mbar_wait(&s.wfree[st1], (fph >> st1) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      fph ^= (1u << st0) | (int4 ? 1u << st1 : 0u);
      const uint8_t* qs = s.q_st + q * s.qslot;
      const __half* scs = reinterpret_cast<const __half*>(s.q_sc + q * s.qscale);
      const uint32_t w0 = smem_u32(s.w_st + st0 * s.wstage);
      const uint32_t w1 = smem_u32(s.w_st + st1 * s.wstage);
      uint4 code[kMaxItems];
      float sc[kMaxItems];
#pragma unroll
      for (int i = 0; i < kMaxItems; ++i) {
        const int it = dtid + i * kDequantThreads;
        if (it < items) {
          code[i] = *reinterpret_cast<const uint4*>(qs + it * 16);  // row it/4, quarter it%4
          sc[i] = __half2float(scs[it >> 2]);
        }
      }
#pragma unroll
      for (int i = 0; i < kMaxItems; ++i) {
        const int it = dtid + i * kDequantThreads;
        if (it >= items) break;
        const int r = it >> 2, qq = it & 3;
        const uint64_t s2 = f32x2(sc[i]), c2 = f32x2(-off * sc[i]);
        const uint32_t wv[4] = {code[i].x, code[i].y, code[i].z, code[i].w};
        const uint32_t rbase = (uint32_t)r * 128;
        if (int4) {
          // elements 32 qq .. 32 qq + 31 of the group: k-block half qq / 2,
          // chunks 4 (qq % 2) .. + 3; word j holds chunk j's 8 nibbles
          const uint32_t dst = ((qq >> 1) ? w1 : w0) + rbase;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t lo = wv[j] & 0x0F0F0F0Fu, hi = (wv[j] >> 4) & 0x0F0F0F0Fu;
            const int c = (qq & 1) * 4 + j;
            st_shared_v4(dst + ((c ^ (r & 7)) << 4), deq2(lo, sel_byte(0), hi, sel_byte(0), s2, c2),
                         deq2(lo, sel_byte(1), hi, sel_byte(1), s2, c2),
                         deq2(lo, sel_byte(2), hi, sel_byte(2), s2, c2),
                         deq2(lo, sel_byte(3), hi, sel_byte(3), s2, c2));
          }
        } else {
          // elements 16 qq .. 16 qq + 15 of the k-block: chunks 2 qq, 2 qq + 1
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t a = wv[2 * j] ^ flip, b = wv[2 * j + 1] ^ flip;
            const int c = qq * 2 + j;
            st_shared_v4(w0 + rbase + ((c ^ (r & 7)) << 4),
                         deq2(a, sel_byte(0), a, sel_byte(1), s2, c2),
                         deq2(a, sel_byte(2), a, sel_byte(3), s2, c2),
                         deq2(b, sel_byte(0), b, sel_byte(1), s2, c2),
                         deq2(b, sel_byte(2), b, sel_byte(3), s2, c2));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {  // one arrival per dequant warp and stage
        mbar_arrive(&s.full[st0]);
        if (int4) mbar_arrive(&s.full[st1]);
        mbar_arrive(&s.qempty[q]);
      }
      advance(q, qph, nq);
    }
    if (!ok) break;
  }
  if (!ok) give_up(s);
}

// ---------------------------------------------------------------- epilogue --

template <bool kSwap, bool kFma>
__device__ void epilogue(const Params& p, const Smem& s, uint32_t tmem) {
  const uint32_t acc_cols = p.acc_stride;
  volatile int* abort_flag = s.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
  uint32_t us = 0, uph = 0, ebuf = 0, xph = 0;
  uint32_t eph[2] = {0, 0};
  bool ok = true;
  int tseq = 0;
  const bool tracer = warp == 4 && lane == 0;
  (void)tseq;
  (void)tracer;
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!(un.flags & kUnitValid)) break;
    const bool gu = unit_gu(un);
    if (kSwap && unit_fma<kFma>(un)) {  // the dequant warps store and publish its rows
      ++tseq;
      continue;
    }
    if (!mbar_wait(&s.accfull[ebuf], eph[ebuf], abort_flag)) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (tracer) FFN_TRACE_SET(tseq, kTrEpiBeg, FFN_TRACE_NS());
    const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + ebuf * acc_cols;
    if (kSwap) {
      const int wr = quarter * 32 + lane;  // weight row of the unit (TMEM lane)
      const int n_pad = max(16, (un.nrows + 15) & ~15);
      if (gu) {
        // lanes 0-63: gate rows, lanes 64-127: the matching up rows
        if (quarter >= 2) {
          if (!mbar_wait(s.xempty, xph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          for (int n0 = 0; n0 < n_pad; n0 += 16) {
            uint32_t u[16];
            tmem_ld16(tb + n0, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) s.xbuf[(n0 + j) * 64 + (wr - 64)] = __uint_as_float(u[j]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(s.xfull);
        } else {
          if (!mbar_wait(s.xfull, xph, abort_flag)) {
            ok = false;
            break;
          }
          for (int n0 = 0; n0 < n_pad; n0 += 16) {
            uint32_t gv[16];
            tmem_ld16(tb + n0, gv);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n0 + j < un.nrows)
                p.h[(size_t)(un.row0 + n0 + j) * p.I + un.wrow0 + wr] = __float2bfloat16_rn(
                    silu_mul(__uint_as_float(gv[j]), s.xbuf[(n0 + j) * 64 + wr]));
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(s.xempty);
        }
        xph ^= 1u;
      } else {
        for (int n0 = 0; n0 < n_pad; n0 += 16) {
          uint32_t v[16];
          tmem_ld16(tb + n0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (n0 + j < un.nrows && wr < un.nbox * kBoxRows)
              p.y[(size_t)(un.row0 + n0 + j) * p.H + un.wrow0 + wr] =
                  __float2bfloat16_rn(__uint_as_float(v[j]));
        }
      }
    } else {
      // D columns follow the weight rows of the stage: gate/up boxes hold 64
      // gate rows then the same 64 up rows, so column 128 c + j (j < 64) pairs
      // with 128 c + 64 + j and is feature wrow0 + 64 c + j.
      const int m = quarter * 32 + lane;  // token row inside the tile
      const bool valid = m < un.nrows;
      if (quarter * 32 < un.nrows) {      // warps holding no row of the tile skip
        __nv_bfloat16* out = gu ? p.h + (size_t)(un.row0 + m) * p.I + un.wrow0
                                : p.y + (size_t)(un.row0 + m) * p.H + un.wrow0;
        uint4* dst = reinterpret_cast<uint4*>(out);
        const int ncols = gu ? un.nbox * (kBoxRows / 2) : un.nbox * kBoxRows;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          uint32_t a[16], b[16];
          const uint32_t col = gu ? (c0 / 64) * 128 + (c0 % 64) : c0;
          tmem_ld16(tb + col, a);
          if (gu) tmem_ld16(tb + col + 64, b);
          tmem_ld_wait();
          float f[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            f[j] = gu ? silu_mul(__uint_as_float(a[j]), __uint_as_float(b[j])) : __uint_as_float(a[j]);
          if (valid) {
            dst[c0 / 8] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
            dst[c0 / 8 + 1] = make_uint4(pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                                         pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.accempty[ebuf]);
    const long long cp = FFN_CLOCK();
    (void)cp;
    if (gu) publish_rows(p, un, lane);
    if (tracer) {
      FFN_TRACE_SET(tseq, kTrEpiEnd, FFN_TRACE_NS());
      FFN_TRACE_SET(tseq, kTrPublish, FFN_CLOCK() - cp);
    }
    ++tseq;
    eph[ebuf] ^= 1u;
    ebuf ^= 1u;
  }
  if (!ok) give_up(s, 6, tseq);
}

// ------------------------------------------------------------------ kernel --
template <bool kSwap, bool kFma>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_ffn_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_h,
                       const __grid_constant__ CUtensorMap tm_xf,
                       const __grid_constant__ CUtensorMap tm_hf, const Params p) {
  extern __shared__ uint8_t ffn_smem_raw[];
  FFN_KSTAMP(0);
  const Smem s = carve(ffn_smem_raw, p, kSwap);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  {  // barrier initialisation, one barrier (set) per thread of warps 2 and 3
    constexpr int kAccInit = kMaxNS + kMaxNQ, kUnitInit = kAccInit + 2;
    static_assert(kUnitInit + kUR < 64, "barrier initialisation needs more threads");
    const int i = threadIdx.x - 64;
    if (i >= 0 && i < kMaxNS) {
      // producer's arrive.expect_tx, then one arrival per dequant warp (INT8/INT4
      // positions) or kDequantWarps more from the producer (BF16 positions)
      mbar_init(&s.full[i], 1 + kDequantWarps);
      mbar_init(&s.empty[i], 1);               // tcgen05.commit (tensor-core positions)
      mbar_init(&s.wfree[i], 1);               // producer, at INT8/INT4 tensor-core positions
      mbar_init(&s.fdone[i], kDequantWarps);   // each dequant warp (CUDA-core positions)
      mbar_init(&s.ffull[i], 1);               // producer's expect_tx, at CUDA-core positions
    } else if (i >= kMaxNS && i < kMaxNS + kMaxNQ) {
      mbar_init(&s.qfull[i - kMaxNS], 1);
      mbar_init(&s.qempty[i - kMaxNS], kDequantWarps);
    } else if (i >= kAccInit && i < kAccInit + 2) {
      mbar_init(&s.accfull[i - kAccInit], 1);
      mbar_init(&s.accempty[i - kAccInit], 4);
    } else if (i >= kUnitInit && i < kUnitInit + kUR) {
      mbar_init(&s.ufull[i - kUnitInit], 1);
      // producer, MMA, code producer, 4 epilogue warps, dequant warps
      mbar_init(&s.uempty[i - kUnitInit], 3 + 4 + kDequantWarps);
    } else if (i == kUnitInit + kUR) {
      mbar_init(s.mmadone, 1);
      mbar_init(s.xfull, 2);   // the two epilogue warps holding the up half
      mbar_init(s.xempty, 2);  // the two epilogue warps holding the gate half
      mbar_init(s.go, 1);      // producer: reserve the next unit
      *s.abort_flag = 0;
    }
    if (i >= 0 && i < 64) fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  const int my_prec = (int)threadIdx.x < p.E ? p.prec[threadIdx.x] : -1;
  pdl_launch_dependents();
  FFN_KSTAMP(1);
  pdl_wait();           // inputs of the previous kernels are complete from here on
  build_entries<kSwap, kFma>(p, s, my_prec);  // contains a __syncthreads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  FFN_KSTAMP(2);
  const uint32_t tmem = *s.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer<kSwap, kFma>(&tm_x, &tm_h, &tm_xf, &tm_hf, p, s);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<kSwap, kFma>(p, s, tmem);
  } else if (warp >= 4 && warp < 8) {
    epilogue<kSwap, kFma>(p, s, tmem);
  } else if (warp == 14) {
    if (lane == 0) code_producer<kFma>(p, s);
  } else if (warp == 15) {
    if (lane == 0) scheduler<kSwap, kFma>(p, s);
  } else {
    if (kSwap) {
      dequant_swap<kFma>(p, s);
    } else {
      const int dtid = (warp < 4 ? warp - 2 : warp - 6) * 32 + lane;  // warps 2, 3, 8 .. 13
      dequant(p, s, dtid);
    }
  }

  FFN_KSTAMP(3);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  FFN_KSTAMP(4);
}

// Stream-ordered swap of a layer's whole descriptor table to a hot set (the
// DynaExq abstract's asynchronous promotion through stable expert handles):
// expert e gets the descriptor of BF16 slot slot_base + i if e == hot_ids[i]
// (hot_ids ascending, n entries), else its base version (the one installed by
// moe_set_expert_precision).  One CTA per expert.  The weights behind every
// descriptor must be complete before this kernel runs (stream order).
__global__ void apply_hot_set_kernel(ExpertDesc* __restrict__ descs, int* __restrict__ prec,
                                     const ExpertDesc* __restrict__ base,
                                     const ExpertDesc* __restrict__ slots,
                                     const int32_t* __restrict__ hot_ids, int n, int slot_base) {
  const int e = blockIdx.x;
  int lo = 0, hi = n;  // first index with hot_ids[index] >= e
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (hot_ids[mid] < e)
      lo = mid + 1;
    else
      hi = mid;
  }
  const bool hot = lo < n && hot_ids[lo] == e;
  const ExpertDesc* src = hot ? slots + slot_base + lo : base + e;
  for (int v = threadIdx.x; v < (int)(sizeof(ExpertDesc) / 16); v += blockDim.x)
    reinterpret_cast<uint4*>(descs + e)[v] = reinterpret_cast<const uint4*>(src)[v];
  if (threadIdx.x == 0) prec[e] = src->prec;
  tmap_release();
}

// Stream-ordered install of one expert descriptor (a by-value kernel argument,
// so the host buffer needs no lifetime beyond the launch) and of its precision
// in the compact precision array.
// dst2 (optional): a second copy (the layer's base table).
__global__ void write_desc_kernel(ExpertDesc* dst, int* prec_dst, ExpertDesc* dst2,
                                  const __grid_constant__ ExpertDesc d) {
  const int i = threadIdx.x;
  for (int v = i; v < (int)(sizeof(ExpertDesc) / 16); v += blockDim.x) {
    reinterpret_cast<uint4*>(dst)[v] = reinterpret_cast<const uint4*>(&d)[v];
    if (dst2 != nullptr) reinterpret_cast<uint4*>(dst2)[v] = reinterpret_cast<const uint4*>(&d)[v];
  }
  if (i == 0) *prec_dst = d.prec;
  tmap_release();
}

}  // namespace ffn
}  // namespace moe
