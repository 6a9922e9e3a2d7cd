// grouped_ffn.cuh -- mixed-precision grouped SwiGLU expert FFN for sm_100a.
//
// One launch computes, for every expert e and every permuted row r of e,
// either the fused gate/up projection with the SwiGLU epilogue
//     h_r = silu(x_r W_g,e^T) * (x_r W_u,e^T)
// or the down projection  y_r = h_r W_d,e^T  (ExactMoE, Section 3.4: "one
// fused gate/up projection and one down projection" per group of experts).
// Experts in one launch may be BF16, INT8 or INT4 (MxMoE abstract: GEMMs of
// different precisions in one grouped kernel); INT8/INT4 weights are
// dequantised to bf16 (q * s, rounded once) in registers inside the mainloop,
// so no bf16 copy of an expert is ever written to global memory (ExactMoE
// Section 3.1: the dequantised values define the operations; no FP16 expert is
// materialised).
//
// Design (one persistent CTA per SM, 12 warps):
//   warp 0  scheduler + TMA producer: takes work units from a global counter
//           in descending cost class (BF16, then INT8, then INT4 experts),
//           streams X tiles and BF16 weight tiles with TMA, INT8/INT4 packed
//           tiles and their fp16 scales into a staging ring.
//   warp 1  TMEM owner + MMA issuer: tcgen05.mma kind::f16, fp32 accumulators
//           in TMEM, double-buffered so the epilogue overlaps the next unit.
//   warps 4-7   epilogue: tcgen05.ld, SwiGLU (gate/up) or copy (down),
//               bf16 stores.
//   warps 8-11  dequant: staged INT8/INT4 codes x fp16 scale -> bf16 in the
//               128-byte-swizzled K-major layout the tensor core reads.
// A work unit is (expert, block of 256 weight rows, tile of <=128 rows).  For
// gate/up the 256 weight rows are 128 gate rows and the matching 128 up rows,
// so the epilogue sees g and u of the same feature.
//
// Two MMA orientations:
//   tile mode (kSwap = false, large groups): A = 128 token rows, B = 256 weight
//     rows, D = 128 x 256 in TMEM; lane = token row.
//   swap mode (kSwap = true, small groups, decode): A = 128 weight rows (two
//     MMAs, one per half), B = the group's rows padded to 16, D = 2 x
//     (128 x N); lane = weight row.  The tensor core then does no work on
//     padding rows, so decode stays bound by weight bytes.
#pragma once

#include "common.cuh"

namespace moe {
namespace ffn {

constexpr int kThreads = 384;
constexpr int kNS = 3;                 // operand stages (64 K-elements each)
constexpr int kNQ = 4;                 // staging slots for packed weights
constexpr int kUR = 4;                 // work-unit ring depth
constexpr int kWStage = 256 * 128;     // 256 weight rows x 128 B (64 bf16)
constexpr int kXStage = 128 * 128;     // 128 rows x 128 B
constexpr int kQSlot = 256 * 64;       // 256 rows x 64 B of packed codes
constexpr int kQScale = 256 * 2;       // 256 fp16 scales
constexpr int kMaxE = 512;
constexpr uint32_t kTmemCols = 512;

struct alignas(64) ExpertDesc {
  CUtensorMap tm_w13;  // codes/values of [2I][H]; box 128 rows x (64 bf16 | 64 B)
  CUtensorMap tm_w2;   // codes/values of [H][I]
  const __half* s13;   // [H/128][2I]
  const __half* s2;    // [I/128][H]
  int prec;            // MOE_BF16 / MOE_INT8 / MOE_INT4, -1 when unset
  int pad[11];
};
static_assert(sizeof(ExpertDesc) == 320, "descriptor layout");

struct Unit {
  int e, prec, wrow0, nwh;  // expert, precision, first weight row, 128-row halves
  int row0, nrows, valid, pad;
};

struct Entry {
  int unit_begin;  // first unit index of this expert
  int e;
  int row0;        // first permuted row of the expert
  int nrows;
};

struct Params {
  const ExpertDesc* descs;
  const int32_t* offsets;  // [E+1]
  __nv_bfloat16* out;      // h (gate/up) or y (down)
  int* counter;            // work counter, zero at launch
  int E, H, I;
  int K;          // reduction length: H (gate/up) or I (down)
  int out_ld;     // row stride of out: I (gate/up) or H (down)
  int n_wblocks;  // I/128 (gate/up) or ceil(H/256) (down)
  int xbox_rows;  // rows per X tensor-map box: 128 (tile mode) or 16 (swap mode)
};

struct Smem {
  uint8_t* w_st;
  uint8_t* x_st;
  uint8_t* q_st;
  uint8_t* q_sc;
  uint64_t *full, *wfull, *empty, *qfull, *qempty, *accfull, *accempty, *ufull, *uempty, *mmadone;
  Unit* units;
  uint32_t* tmem_slot;
  int* abort_flag;
  int* n_entries;
  int* n_units;
  Entry* entries;
};

__host__ __device__ constexpr size_t smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)kNS * kWStage + (size_t)kNS * kXStage +
         (size_t)kNQ * kQSlot + (size_t)kNQ * kQScale + 64 * sizeof(uint64_t) /* barriers */ +
         kUR * sizeof(Unit) + 64 /* misc words */ + (size_t)kMaxE * sizeof(Entry);
}

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.w_st = p;
  p += kNS * kWStage;
  s.x_st = p;
  p += kNS * kXStage;
  s.q_st = p;
  p += kNQ * kQSlot;
  s.q_sc = p;
  p += kNQ * kQScale;
  uint64_t* b = reinterpret_cast<uint64_t*>(p);
  s.full = b;
  s.wfull = s.full + kNS;
  s.empty = s.wfull + kNS;
  s.qfull = s.empty + kNS;
  s.qempty = s.qfull + kNQ;
  s.accfull = s.qempty + kNQ;
  s.accempty = s.accfull + 2;
  s.ufull = s.accempty + 2;
  s.uempty = s.ufull + kUR;
  s.mmadone = s.uempty + kUR;
  p += 64 * sizeof(uint64_t);
  s.units = reinterpret_cast<Unit*>(p);
  p += kUR * sizeof(Unit);
  s.tmem_slot = reinterpret_cast<uint32_t*>(p);
  s.abort_flag = reinterpret_cast<int*>(p + 4);
  s.n_entries = reinterpret_cast<int*>(p + 8);
  s.n_units = reinterpret_cast<int*>(p + 12);
  p += 64;
  s.entries = reinterpret_cast<Entry*>(p);
  return s;
}

__device__ __forceinline__ void advance(uint32_t& slot, uint32_t& phase, uint32_t n) {
  if (++slot == n) {
    slot = 0;
    phase ^= 1u;
  }
}

__device__ __forceinline__ void give_up(const Smem& s) {
  *reinterpret_cast<volatile int*>(s.abort_flag) = 1;
  flag_status(MOE_STATUS_WAIT_TIMEOUT);
}

// Work units of one expert with n rows.
__device__ __forceinline__ int units_of(int n, int n_wblocks) {
  return n > 0 ? ((n + 127) / 128) * n_wblocks : 0;
}

// Warp 0: list the experts with rows, cheapest-last (BF16 < INT8 < INT4 in
// precision code = descending bytes per weight), with their first unit index.
__device__ void build_entries(const Params& p, const Smem& s) {
  const int lane = threadIdx.x & 31;
  const int per = (p.E + 31) / 32;
  const int e0 = lane * per;
  int unit_run = 0, ent_run = 0;
  bool unset = false;
  for (int cls = MOE_BF16; cls <= MOE_INT4; ++cls) {
    int my_units = 0, my_ents = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e >= p.E) break;
      const int n = p.offsets[e + 1] - p.offsets[e];
      const int prec = p.descs[e].prec;
      if (cls == MOE_BF16 && n > 0 && (prec < MOE_BF16 || prec > MOE_INT4)) unset = true;
      if (prec == cls && n > 0) {
        my_units += units_of(n, p.n_wblocks);
        my_ents += 1;
      }
    }
    int u_incl = my_units, e_incl = my_ents;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, u_incl, d);
      const int b = __shfl_up_sync(0xffffffffu, e_incl, d);
      if (lane >= d) {
        u_incl += a;
        e_incl += b;
      }
    }
    int u = unit_run + u_incl - my_units, en = ent_run + e_incl - my_ents;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e >= p.E) break;
      const int n = p.offsets[e + 1] - p.offsets[e];
      if (p.descs[e].prec == cls && n > 0) {
        s.entries[en] = Entry{u, e, p.offsets[e], n};
        u += units_of(n, p.n_wblocks);
        en += 1;
      }
    }
    unit_run += __shfl_sync(0xffffffffu, u_incl, 31);
    ent_run += __shfl_sync(0xffffffffu, e_incl, 31);
  }
  if (__any_sync(0xffffffffu, unset) && lane == 0) flag_status(MOE_STATUS_UNSET_EXPERT);
  if (lane == 0) {
    *s.n_units = unit_run;
    *s.n_entries = ent_run;
  }
}

template <bool kGateUp>
__device__ __forceinline__ Unit decode_unit(const Params& p, const Smem& s, int u) {
  int lo = 0, hi = *s.n_entries - 1;  // last entry with unit_begin <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.entries[mid].unit_begin <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  const Entry en = s.entries[lo];
  const int local = u - en.unit_begin;
  const int tt = local / p.n_wblocks, wb = local % p.n_wblocks;
  Unit un;
  un.e = en.e;
  un.prec = p.descs[en.e].prec;
  un.row0 = en.row0 + tt * 128;
  un.nrows = min(128, en.nrows - tt * 128);
  if (kGateUp) {
    un.wrow0 = wb * 128;
    un.nwh = 2;
  } else {
    un.wrow0 = wb * 256;
    un.nwh = min(2, (p.H - un.wrow0) / 128);
  }
  un.valid = 1;
  un.pad = 0;
  return un;
}

template <bool kGateUp>
__device__ __forceinline__ int weight_row(const Params& p, const Unit& un, int h) {
  return kGateUp ? (h == 0 ? un.wrow0 : p.I + un.wrow0) : un.wrow0 + 128 * h;
}

// ---------------------------------------------------------------- producer --
template <bool kGateUp, bool kSwap>
__device__ void producer(const CUtensorMap* tm_x, const Params& p, const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  uint32_t st = 0, sph = 0, q = 0, qph = 0, us = 0, uph = 0;
  uint32_t issued = 0, issued_par = 0, qissued = 0, qissued_par = 0;  // drain bookkeeping
  const int total = *s.n_units;
  const int nkb = p.K / 64;
  bool ok = true;
  prefetch_tmap(tm_x);
  for (;;) {
    if (!mbar_wait(&s.uempty[us], uph ^ 1u, abort_flag)) {
      ok = false;
      break;
    }
    const int u = atomicAdd(p.counter, 1);
    Unit un;
    if (u < total) {
      un = decode_unit<kGateUp>(p, s, u);
    } else {
      un = Unit{0, 0, 0, 0, 0, 0, 0, 0};
    }
    s.units[us] = un;
    mbar_arrive(&s.ufull[us]);
    advance(us, uph, kUR);
    if (!un.valid) break;

    const ExpertDesc* d = p.descs + un.e;
    const CUtensorMap* tw = kGateUp ? &d->tm_w13 : &d->tm_w2;
    const __half* sc = kGateUp ? d->s13 : d->s2;
    const int srows = kGateUp ? 2 * p.I : p.H;  // rows of the scale matrix
    tmap_acquire(tw);
    prefetch_tmap(tw);
    const int nxb = kSwap ? (un.nrows + p.xbox_rows - 1) / p.xbox_rows : 1;
    const uint32_t xbytes = (uint32_t)(nxb * p.xbox_rows * 128);
    for (int kb = 0; kb < nkb && ok; ++kb) {
      if (!mbar_wait(&s.empty[st], sph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      if (un.prec != MOE_BF16 && (un.prec == MOE_INT8 || (kb & 1) == 0)) {
        if (!mbar_wait(&s.qempty[q], qph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&s.qfull[q], (uint32_t)un.nwh * (128 * 64 + 256));
        const int kc = (un.prec == MOE_INT8) ? kb * 64 : (kb >> 1) * 64;  // byte column
        const int g = kb >> 1;                                             // K-group
        for (int h = 0; h < un.nwh; ++h) {
          const int wr = weight_row<kGateUp>(p, un, h);
          tma_load_2d(s.q_st + q * kQSlot + h * 8192, tw, kc, wr, &s.qfull[q]);
          bulk_load(s.q_sc + q * kQScale + h * 256, sc + (size_t)g * srows + wr, 256, &s.qfull[q]);
        }
        qissued |= 1u << q;
        qissued_par = (qissued_par & ~(1u << q)) | (qph << q);
        advance(q, qph, kNQ);
      }
      const uint32_t bytes = xbytes + (un.prec == MOE_BF16 ? (uint32_t)un.nwh * 16384u : 0u);
      mbar_arrive_expect_tx(&s.full[st], bytes);
      for (int b = 0; b < nxb; ++b)
        tma_load_2d(s.x_st + st * kXStage + b * p.xbox_rows * 128, tm_x, kb * 64,
                    un.row0 + b * p.xbox_rows, &s.full[st]);
      if (un.prec == MOE_BF16)
        for (int h = 0; h < un.nwh; ++h)
          tma_load_2d(s.w_st + st * kWStage + h * 16384, tw, kb * 64, weight_row<kGateUp>(p, un, h),
                      &s.full[st]);
      issued |= 1u << st;
      issued_par = (issued_par & ~(1u << st)) | (sph << st);
      advance(st, sph, kNS);
    }
    if (!ok) break;
  }
  if (!ok) {
    give_up(s);
    // Let copies already in flight land before the CTA's shared memory goes away.
    for (uint32_t i = 0; i < (uint32_t)kNS; ++i)
      if (issued & (1u << i)) mbar_wait(&s.full[i], (issued_par >> i) & 1u);
    for (uint32_t i = 0; i < (uint32_t)kNQ; ++i)
      if (qissued & (1u << i)) mbar_wait(&s.qfull[i], (qissued_par >> i) & 1u);
  }
}

// -------------------------------------------------------------- MMA issuer --
template <bool kGateUp, bool kSwap>
__device__ void mma_issuer(const Params& p, const Smem& s, uint32_t tmem) {
  volatile int* abort_flag = s.abort_flag;
  uint32_t st = 0, sph = 0, us = 0, uph = 0, abuf = 0;
  uint32_t aph[2] = {0, 0};
  uint32_t wph = 0;  // wfull phase bit per stage: it only advances on INT8/INT4 units
  const int nkb = p.K / 64;
  bool ok = true;
  for (;;) {
    if (!mbar_wait(&s.ufull[us], uph, abort_flag)) {
      ok = false;
      break;
    }
    const Unit un = s.units[us];
    mbar_arrive(&s.uempty[us]);
    advance(us, uph, kUR);
    if (!un.valid) break;
    if (!mbar_wait(&s.accempty[abuf], aph[abuf] ^ 1u, abort_flag)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d_base = tmem + abuf * 256;
    const int nmma = kSwap ? max(16, (un.nrows + 15) & ~15) : un.nwh * 128;
    const uint32_t idesc = idesc_bf16_f32(128, nmma);
    const bool quant = un.prec != MOE_BF16;
    for (int kb = 0; kb < nkb; ++kb) {
      if (!mbar_wait(&s.full[st], sph, abort_flag) ||
          (quant && !mbar_wait(&s.wfull[st], (wph >> st) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      if (quant) wph ^= 1u << st;
      tc_fence_after();
      const uint32_t xa = smem_u32(s.x_st + st * kXStage);
      const uint32_t wa = smem_u32(s.w_st + st * kWStage);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (kb | kk) != 0;
        if (kSwap) {
          for (int h = 0; h < un.nwh; ++h)
            mma_bf16_ss(d_base + h * 128, smem_desc_sw128(wa + h * 16384 + kk * 32),
                        smem_desc_sw128(xa + kk * 32), idesc, acc);
        } else {
          mma_bf16_ss(d_base, smem_desc_sw128(xa + kk * 32), smem_desc_sw128(wa + kk * 32), idesc,
                      acc);
        }
      }
      mma_commit(&s.empty[st]);
      advance(st, sph, kNS);
    }
    if (!ok) break;
    mma_commit(&s.accfull[abuf]);
    aph[abuf] ^= 1u;
    abuf ^= 1u;
  }
  if (!ok) give_up(s);
  // All issued MMAs must finish before TMEM is released.
  mma_commit(s.mmadone);
  mbar_wait(s.mmadone, 0);
}

// ----------------------------------------------------------------- dequant --
// 128 threads convert one 64-element K-slice of up to 256 weight rows: thread
// (row r = tid/8 + 16 i, 16-byte chunk c = tid % 8) -> 8 bf16 at the swizzled
// position of chunk c in row r.  Each warp signals its own part (barrier
// counts are 4), so the four warps never wait on one another.
template <bool kGateUp>
__device__ void dequant(const Params& p, const Smem& s) {
  volatile int* abort_flag = s.abort_flag;
  const int tid = threadIdx.x - 256;  // 0..127
  const int lane = threadIdx.x & 31;
  const int c = tid & 7, rsub = tid >> 3;
  uint32_t st = 0, sph = 0, q = 0, qph = 0, us = 0, uph = 0;
  const int nkb = p.K / 64;
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
    if (!un.valid) break;
    if (un.prec == MOE_BF16) {
      for (int kb = 0; kb < nkb; ++kb) advance(st, sph, kNS);
      continue;
    }
    const int rows = un.nwh * 128;
    for (int kb = 0; kb < nkb; ++kb) {
      const bool first = un.prec == MOE_INT8 || (kb & 1) == 0;
      const bool last = un.prec == MOE_INT8 || (kb & 1) == 1;
      if ((first && !mbar_wait(&s.qfull[q], qph, abort_flag)) ||
          !mbar_wait(&s.empty[st], sph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const uint8_t* qs = s.q_st + q * kQSlot;
      const __half* scs = reinterpret_cast<const __half*>(s.q_sc + q * kQScale);
      const uint32_t wdst = smem_u32(s.w_st + st * kWStage);
      for (int r = rsub; r < rows; r += 16) {
        const int h = r >> 7, rr = r & 127;
        const float sc = __half2float(scs[h * 128 + rr]);
        const uint8_t* src = qs + h * 8192 + rr * 64;
        float f[8];
        if (un.prec == MOE_INT4) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(src + (kb & 1) * 32 + c * 4);
#pragma unroll
          for (int j = 0; j < 8; ++j)  // (2^23 + u) - (2^23 + 8) = u - 8 = q, exact
            f[j] = (__uint_as_float(0x4B000000u | ((v >> (4 * j)) & 0xFu)) - 8388616.0f) * sc;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(src + c * 8);
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // (2^23 + q + 128) - (2^23 + 128) = q, exact
            const uint32_t b = ((j < 4 ? v.x : v.y) >> (8 * (j & 3))) & 0xFFu;
            f[j] = (__uint_as_float(0x4B000000u | (b ^ 0x80u)) - 8388736.0f) * sc;
          }
        }
        st_shared_v4(wdst + r * 128 + ((c ^ (r & 7)) << 4), pack_bf16x2(f[0], f[1]),
                     pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {  // one arrival per dequant warp (barrier counts are 4)
        mbar_arrive(&s.wfull[st]);
        if (last) mbar_arrive(&s.qempty[q]);
      }
      if (last) advance(q, qph, kNQ);
      advance(st, sph, kNS);
    }
    if (!ok) break;
  }
  if (!ok) give_up(s);
}

// ---------------------------------------------------------------- epilogue --
__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

template <bool kGateUp, bool kSwap>
__device__ void epilogue(const Params& p, const Smem& s, uint32_t tmem) {
  volatile int* abort_flag = s.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
  uint32_t us = 0, uph = 0, ebuf = 0;
  uint32_t eph[2] = {0, 0};
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
    if (!un.valid) break;
    if (!mbar_wait(&s.accfull[ebuf], eph[ebuf], abort_flag)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + ebuf * 256;
    if (kSwap) {
      const int wr = quarter * 32 + lane;  // weight row inside a 128-row half
      const int n_pad = max(16, (un.nrows + 15) & ~15);
      for (int n0 = 0; n0 < n_pad; n0 += 16) {
        if (kGateUp) {
          uint32_t g[16], u[16];
          tmem_ld16(tb + n0, g);
          tmem_ld16(tb + 128 + n0, u);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (n0 + j < un.nrows)
              p.out[(size_t)(un.row0 + n0 + j) * p.out_ld + un.wrow0 + wr] =
                  __float2bfloat16_rn(silu_mul(__uint_as_float(g[j]), __uint_as_float(u[j])));
        } else {
          for (int h = 0; h < un.nwh; ++h) {
            uint32_t v[16];
            tmem_ld16(tb + h * 128 + n0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n0 + j < un.nrows)
                p.out[(size_t)(un.row0 + n0 + j) * p.out_ld + un.wrow0 + h * 128 + wr] =
                    __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        }
      }
    } else {
      const int m = quarter * 32 + lane;  // token row inside the tile
      const bool valid = m < un.nrows;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)(un.row0 + m) * p.out_ld + un.wrow0);
      const int ncols = kGateUp ? 128 : un.nwh * 128;
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        uint32_t a[16], b[16];
        tmem_ld16(tb + c0, a);
        if (kGateUp) tmem_ld16(tb + 128 + c0, b);
        tmem_ld_wait();
        float f[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          f[j] = kGateUp ? silu_mul(__uint_as_float(a[j]), __uint_as_float(b[j]))
                         : __uint_as_float(a[j]);
        if (valid) {
          dst[c0 / 8] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                   pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          dst[c0 / 8 + 1] = make_uint4(pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                                       pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.accempty[ebuf]);
    eph[ebuf] ^= 1u;
    ebuf ^= 1u;
  }
  if (!ok) give_up(s);
}

// ------------------------------------------------------------------ kernel --
template <bool kGateUp, bool kSwap>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_ffn_kernel(const __grid_constant__ CUtensorMap tm_x, const Params p) {
  extern __shared__ uint8_t ffn_smem_raw[];
  const Smem s = carve(ffn_smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&s.full[i], 1);   // producer's arrive.expect_tx
      mbar_init(&s.wfull[i], 4);  // one arrival per dequant warp
      mbar_init(&s.empty[i], 1);  // tcgen05.commit
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(&s.qfull[i], 1);
      mbar_init(&s.qempty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.accfull[i], 1);
      mbar_init(&s.accempty[i], 4);
    }
    for (int i = 0; i < kUR; ++i) {
      mbar_init(&s.ufull[i], 1);
      mbar_init(&s.uempty[i], 9);  // MMA thread + 4 epilogue warps + 4 dequant warps
    }
    mbar_init(s.mmadone, 1);
    *s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) build_entries(p, s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer<kGateUp, kSwap>(&tm_x, p, s);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<kGateUp, kSwap>(p, s, tmem);
  } else if (warp >= 4 && warp < 8) {
    epilogue<kGateUp, kSwap>(p, s, tmem);
  } else if (warp >= 8) {
    dequant<kGateUp>(p, s);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Stream-ordered install of one expert descriptor (a by-value kernel argument,
// so the host buffer needs no lifetime beyond the launch).
__global__ void write_desc_kernel(ExpertDesc* dst, const __grid_constant__ ExpertDesc d) {
  const int i = threadIdx.x;
  if (i < (int)(sizeof(ExpertDesc) / 16))
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(&d)[i];
  tmap_release();
}

}  // namespace ffn
}  // namespace moe
