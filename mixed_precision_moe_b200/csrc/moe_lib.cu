// moe_lib.cu -- host side of the libmoe C ABI (include/moe.h) and the single
// translation unit that holds every kernel of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "grouped_ffn.cuh"
#include "route_permute_combine.cuh"
#include "router.cuh"

namespace {
constexpr int kMaxDevices = 64;  // per-device caches below

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return MOE_OK;
}

#define MOE_CUDA_TRY(expr)                                                              \
  do {                                                                                  \
    cudaError_t err_ = (expr);                                                          \
    if (err_ != cudaSuccess)                                                            \
      return fail(MOE_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(err_));      \
  } while (0)

#define MOE_CHECK(cond, code, ...) \
  do {                             \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows][cols] matrix of `esize`-byte elements,
// box = box_rows x box_cols elements.
int encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, int esize,
              uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
              CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  MOE_CHECK(fn != nullptr, MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MOE_CHECK(r == CUDA_SUCCESS, MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOE_OK;
}

// 3-D map over a row-major [d2][rows][cols] array; box = box_d2 x box_rows x
// box_cols elements.
int encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, int esize,
              uint64_t d2, uint64_t rows, uint64_t cols, uint32_t box_d2, uint32_t box_rows,
              uint32_t box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  MOE_CHECK(fn != nullptr, MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {cols, rows, d2};
  cuuint64_t strides[2] = {cols * (uint64_t)esize, rows * cols * (uint64_t)esize};
  cuuint32_t box[3] = {box_cols, box_rows, box_d2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MOE_CHECK(r == CUDA_SUCCESS, MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOE_OK;
}

// Tensor maps of one expert's weights in their storage format.  Every box
// holds 128 weight rows x 64 K-elements, so one TMA fetches a whole 128-row
// operand block:
//   w13 [2I][K] is mapped as [2][I][K] with box 2 x 64 x 64: rows r .. r+63 of
//     the gate half and the same rows of the up half in one copy;
//   w2 [H][K] as a 2-D map with box 128 x 64.
// BF16 values land in the 128-byte-swizzled layout the MMA reads; INT8/INT4
// codes (64 bytes of a row per box) are staged unswizzled and dequantised.
// INT8/INT4 experts also get the maps of the CUDA-core path (layers with H and I
// of at least 256): codes in 128-byte K boxes (128 rows: 64 gate + 64 up rows,
// or 128 down rows) and the fp16 scales of one stage's K-groups (INT4: two,
// INT8: one) for the same rows, the gate/up scales viewed as [G][2][I].
bool fma_capable(int H, int I) { return H >= 256 && I >= 256; }

int encode_weights(moe::ffn::ExpertDesc* d, const moe_expert_weights* w, int prec, int H, int I) {
  const bool bf16 = prec == MOE_BF16;
  const CUtensorMapDataType t = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int es = bf16 ? 2 : 1;
  const CUtensorMapSwizzle swz = bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  const int cols13 = prec == MOE_INT4 ? H / 2 : H, cols2 = prec == MOE_INT4 ? I / 2 : I;
  int rc = encode_3d(&d->tm_w13, w->w13, t, es, 2, I, cols13, 2, 64, 64, swz);
  if (rc != MOE_OK) return rc;
  rc = encode_2d(&d->tm_w2, w->w2, t, es, H, cols2, 128, 64, swz);
  if (rc != MOE_OK || bf16 || !fma_capable(H, I)) return rc;
  const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
  const uint32_t gs = prec == MOE_INT4 ? 2 : 1;  // K-groups per CUDA-core stage
  rc = encode_3d(&d->tm_q13f, w->w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 2, I, cols13, 2, 64, 128,
                 none);
  if (rc != MOE_OK) return rc;
  rc = encode_2d(&d->tm_q2f, w->w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H, cols2, 128, 128, none);
  if (rc != MOE_OK) return rc;
  rc = encode_3d(&d->tm_s13f, w->s13, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, H / 128, 2, I, gs, 2, 64,
                 none);
  if (rc != MOE_OK) return rc;
  rc = encode_2d(&d->tm_s2f, w->s2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, I / 128, H, gs, 128, none);
  if (rc != MOE_OK) return rc;
  // half-height down units (64 rows) of the CUDA-core path
  rc = encode_2d(&d->tm_q2h, w->w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H, cols2, 64, 128, none);
  if (rc != MOE_OK) return rc;
  return encode_2d(&d->tm_s2h, w->s2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, I / 128, H, gs, 64,
                   none);
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor in the stream drains; the kernels themselves execute
// griddepcontrol.wait before reading anything a predecessor wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Scheduler counters at the end of the FFN workspace: the work counters, then
// (from int 16) one gate/up completion counter per expert and the ready list
// of experts ([E]).
constexpr size_t kFfnCounterBytes = 8192;
size_t ffn_counter_bytes(int E) { return (16 + 2 * (size_t)E) * sizeof(int); }
static_assert((16 + 2 * 512) * sizeof(int) <= kFfnCounterBytes, "counter space");

int num_sms(int device) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return 0;
  return n;
}

}  // namespace

struct moe_layer {
  int H, I, E, k;
  int device;
  moe::ffn::ExpertDesc* d_descs;  // [E], device: the table the forwards read
  int* d_prec;                    // [E], device: compact copy of the precisions
  moe::ffn::ExpertDesc* d_base;   // [E], device: the versions installed by set_expert_precision
  moe::ffn::ExpertDesc* d_slots = nullptr;  // [n_slots], device: BF16 promotion slots
  int n_slots = 0;
  unsigned int* hot = nullptr;    // device [E]: selection counts (NULL: not counted)
  std::vector<int> prec;          // host shadow of the base versions, -1 = unset
};

extern "C" {

const char* moe_last_error(void) { return g_last_error.c_str(); }

int moe_abi_version(void) { return 1; }

#ifdef MOE_FFN_TRACE
// Profiling builds only (not part of moe.h): the grouped FFN's per-unit record.
size_t moe_ffn_trace_bytes(void) { return sizeof(moe::ffn::g_ffn_trace); }

int moe_ffn_trace_reset(void) {
  void* addr = nullptr;
  MOE_CUDA_TRY(cudaGetSymbolAddress(&addr, moe::ffn::g_ffn_trace));
  MOE_CUDA_TRY(cudaMemset(addr, 0, sizeof(moe::ffn::g_ffn_trace)));
  return ok();
}

int moe_ffn_giveup_read(int* host_dst, size_t bytes) {
  MOE_CHECK(host_dst != nullptr && bytes <= sizeof(moe::ffn::g_ffn_giveup), MOE_ERR_INVALID_ARG,
            "bad buffer");
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(host_dst, moe::ffn::g_ffn_giveup, bytes));
  static const int zero[moe::ffn::kTraceCtas * 4] = {};
  MOE_CUDA_TRY(cudaMemcpyToSymbol(moe::ffn::g_ffn_giveup, zero, sizeof zero));
  return ok();
}

int moe_ffn_kstamp_read(long long* host_dst, size_t bytes) {
  MOE_CHECK(host_dst != nullptr && bytes <= sizeof(moe::ffn::g_ffn_kstamp), MOE_ERR_INVALID_ARG,
            "bad buffer");
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(host_dst, moe::ffn::g_ffn_kstamp, bytes));
  return ok();
}

int moe_ffn_trace_read(void* host_dst, size_t bytes) {
  MOE_CHECK(host_dst != nullptr && bytes <= sizeof(moe::ffn::g_ffn_trace), MOE_ERR_INVALID_ARG,
            "bad trace buffer");
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(host_dst, moe::ffn::g_ffn_trace, bytes));
  return ok();
}
#endif

int moe_layer_create(int H, int I, int E, int k, moe_layer_t* out) {
  MOE_CHECK(out != nullptr, MOE_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  MOE_CHECK(H > 0 && I > 0 && H % 128 == 0 && I % 128 == 0, MOE_ERR_UNSUPPORTED,
            "H=%d and I=%d must be positive multiples of 128", H, I);
  MOE_CHECK(E >= 1 && E <= moe::ffn::kMaxE, MOE_ERR_UNSUPPORTED, "E=%d outside [1, 512]", E);
  MOE_CHECK(k >= 1 && k <= 16 && k <= E, MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 16)]", k);
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  moe::ffn::ExpertDesc* d = nullptr;
  const size_t table = sizeof(moe::ffn::ExpertDesc) * E;
  // active table, then the base table, then the compact precisions
  MOE_CUDA_TRY(cudaMalloc(&d, 2 * table + sizeof(int) * E));
  int* dp = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(d) + 2 * table);
  // All bytes 0xFF: prec = -1 (unset) for every expert, in every array.
  cudaError_t e1 = cudaMemset(d, 0xFF, 2 * table + sizeof(int) * E);
  cudaError_t e2 = cudaDeviceSynchronize();
  if (e1 != cudaSuccess || e2 != cudaSuccess) {
    cudaFree(d);
    return fail(MOE_ERR_CUDA, "descriptor table init failed: %s",
                cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
  }
  moe_layer* L = new moe_layer{H, I, E, k, dev, d, dp, d + E};
  L->prec.assign(E, -1);
  *out = L;
  return ok();
}

int moe_layer_destroy(moe_layer_t layer) {
  MOE_CHECK(layer != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  cudaDeviceSynchronize();
  cudaError_t e = cudaFree(layer->d_descs);
  if (layer->d_slots != nullptr) cudaFree(layer->d_slots);
  delete layer;
  MOE_CHECK(e == cudaSuccess, MOE_ERR_CUDA, "cudaFree failed: %s", cudaGetErrorString(e));
  return ok();
}

int moe_set_expert_precision(moe_layer_t L, int expert, moe_precision_t precision,
                             const moe_expert_weights* w, void* stream) {
  MOE_CHECK(L != nullptr && w != nullptr, MOE_ERR_INVALID_ARG, "null layer or weights");
  MOE_CHECK(expert >= 0 && expert < L->E, MOE_ERR_INVALID_ARG, "expert %d outside [0, %d)",
            expert, L->E);
  const int prec = (int)precision;
  MOE_CHECK(prec == MOE_BF16 || prec == MOE_INT8 || prec == MOE_INT4, MOE_ERR_INVALID_ARG,
            "unknown precision %d", prec);
  MOE_CHECK(w->w13 != nullptr && w->w2 != nullptr, MOE_ERR_INVALID_ARG, "null weight pointer");
  MOE_CHECK(aligned(w->w13, 16) && aligned(w->w2, 16), MOE_ERR_UNSUPPORTED,
            "weight buffers must be 16-byte aligned");
  if (prec != MOE_BF16) {
    MOE_CHECK(w->s13 != nullptr && w->s2 != nullptr, MOE_ERR_INVALID_ARG,
              "INT8/INT4 experts need scales");
    MOE_CHECK(aligned(w->s13, 16) && aligned(w->s2, 16), MOE_ERR_UNSUPPORTED,
              "scale buffers must be 16-byte aligned");
  }
  moe::ffn::ExpertDesc d;
  memset(&d, 0, sizeof d);
  const int rc = encode_weights(&d, w, prec, L->H, L->I);
  if (rc != MOE_OK) return rc;
  d.s13 = prec == MOE_BF16 ? nullptr : static_cast<const __half*>(w->s13);
  d.s2 = prec == MOE_BF16 ? nullptr : static_cast<const __half*>(w->s2);
  d.prec = prec;
  moe::ffn::write_desc_kernel<<<1, 32, 0, as_stream(stream)>>>(L->d_descs + expert,
                                                               L->d_prec + expert,
                                                               L->d_base + expert, d);
  MOE_CUDA_TRY(cudaGetLastError());
  L->prec[expert] = prec;
  return ok();
}

int moe_get_expert_precision(moe_layer_t L, int expert, int* precision) {
  MOE_CHECK(L != nullptr && precision != nullptr, MOE_ERR_INVALID_ARG, "null argument");
  MOE_CHECK(expert >= 0 && expert < L->E, MOE_ERR_INVALID_ARG, "expert %d outside [0, %d)",
            expert, L->E);
  *precision = L->prec[expert];
  return ok();
}

int moe_route_topk(const float* logits, int T, int E, int k, int renormalize, int32_t* topk_idx,
                   float* topk_w, void* stream) {
  MOE_CHECK(T >= 0, MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  MOE_CHECK(E >= 1 && E <= 512, MOE_ERR_UNSUPPORTED, "E=%d outside [1, 512]", E);
  MOE_CHECK(k >= 1 && k <= 16 && k <= E, MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 16)]", k);
  if (T == 0) return ok();
  MOE_CHECK(logits && topk_idx && topk_w, MOE_ERR_INVALID_ARG, "null pointer");
  const int keys = (E + 31) / 32;
  const dim3 block(256), grid((T + 7) / 8);
  cudaStream_t s = as_stream(stream);
  auto kern = keys <= 1 ? moe::route_topk_kernel<1>
            : keys <= 2 ? moe::route_topk_kernel<2>
            : keys <= 4 ? moe::route_topk_kernel<4>
            : keys <= 8 ? moe::route_topk_kernel<8>
                        : moe::route_topk_kernel<16>;
  MOE_CUDA_TRY(launch_pdl(kern, grid, block, 0, s, logits, T, E, k, renormalize, topk_idx, topk_w));
  return ok();
}

}  // extern "C"

namespace {
// ------------------------------------------------ router projection + top-k --
// Host checks of moe_router_topk's arguments (also run by
// moe_layer_forward_hidden before it enqueues anything).
int router_check(const void* h, const void* w_router, int T, int H, int E, int k, int do_topk,
                 const float* logits, const int32_t* topk_idx, const float* topk_w) {
  MOE_CHECK(T >= 0, MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  MOE_CHECK(H >= moe::router::kKB && H % moe::router::kKB == 0, MOE_ERR_UNSUPPORTED,
            "H=%d must be a positive multiple of %d", H, moe::router::kKB);
  MOE_CHECK(E >= 1 && E <= moe::router::kMaxE, MOE_ERR_UNSUPPORTED, "E=%d outside [1, 512]", E);
  if (do_topk)
    MOE_CHECK(k >= 1 && k <= 16 && k <= E, MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 16)]",
              k);
  MOE_CHECK((T + moe::router::tm_of(E) - 1) / moe::router::tm_of(E) <= 65535,
            MOE_ERR_UNSUPPORTED, "T=%d too large", T);
  if (T == 0) return MOE_OK;
  MOE_CHECK(h && w_router, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(!do_topk || (topk_idx && topk_w), MOE_ERR_INVALID_ARG, "null top-k output");
  MOE_CHECK(do_topk || logits, MOE_ERR_INVALID_ARG, "nothing to write: no logits, no top-k");
  MOE_CHECK(aligned(h, 16) && aligned(w_router, 16), MOE_ERR_UNSUPPORTED,
            "h and w_router must be 16-byte aligned");
  return MOE_OK;
}

// Attributes of router_topk_kernel<KEYS> on the current device, set once: the
// shared-memory limit and clusters of up to 16 CTAs (non-portable).  Returns
// the largest cluster size to use: 16 if a cluster of 16 CTAs with the full
// shared memory fits on this GPU, else 8.
template <int KEYS>
int router_attributes(int dev) {
  static std::atomic<int> max_cluster[kMaxDevices];
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && max_cluster[dev].load() != 0) return max_cluster[dev].load();
  auto kern = moe::router::router_topk_kernel<KEYS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)moe::router::kSmemLimit) != cudaSuccess)
    return 0;
  int m = 8;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16);
    cfg.blockDim = dim3(moe::router::kThreads);
    cfg.dynamicSmemBytes = moe::router::kSmemLimit;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1) m = 16;
  }
  cudaGetLastError();  // a refused attribute or query leaves no sticky error
  if (cached) max_cluster[dev].store(m);
  return m;
}

template <int KEYS>
int router_launch(const CUtensorMap& tm_h, const CUtensorMap& tm_w, const moe::router::Params& prm,
                  int S, int tiles, size_t smem, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, tiles);
  cfg.blockDim = dim3(moe::router::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, moe::router::router_topk_kernel<KEYS>, tm_h, tm_w, prm));
  return MOE_OK;
}

// z = W_r h on the tensor cores, then (do_topk) the top-k of every token.
// Cluster size S: the largest power of two <= 16 (8 where a 16-CTA cluster
// does not fit; and <= H / 64) that keeps
// tiles * S within the SM count; stages: as many as the shared memory holds,
// up to the k-blocks of one CTA.
int router_impl(const void* h, const void* w_router, int T, int H, int E, int k, int renormalize,
                int do_topk, float* logits, int32_t* topk_idx, float* topk_w, void* stream) {
  namespace R = moe::router;
  int rc = router_check(h, w_router, T, H, E, k, do_topk, logits, topk_idx, topk_w);
  if (rc != MOE_OK || T == 0) return rc;
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  const int npad = R::npad_of(E), tm = R::tm_of(E), nkb = H / R::kKB;
  const int tiles = (T + tm - 1) / tm;
  const int nsm = std::max(1, num_sms(dev));
  const int keys = (E + 31) / 32;
  const int max_cluster = keys <= 1   ? router_attributes<1>(dev)
                          : keys <= 2 ? router_attributes<2>(dev)
                          : keys <= 4 ? router_attributes<4>(dev)
                          : keys <= 8 ? router_attributes<8>(dev)
                                      : router_attributes<16>(dev);
  MOE_CHECK(max_cluster > 0, MOE_ERR_CUDA, "cannot set the router kernel's attributes");
  int S = 1;
  while (S * 2 <= max_cluster && S * 2 <= nkb && tiles * S * 2 <= nsm) S *= 2;
  const int nkl_max = (nkb + S - 1) / S;
  int ns = 1;
  while (ns < nkl_max && R::layout(npad, tm, ns + 1, S).total <= R::kSmemLimit) ++ns;
  const size_t smem = R::layout(npad, tm, ns, S).total;
  MOE_CHECK(smem <= R::kSmemLimit, MOE_ERR_UNSUPPORTED, "router tile does not fit (E=%d)", E);
  CUtensorMap tm_h, tm_w;
  const int hrows = std::min(tm, (T + 7) / 8 * 8);
  rc = encode_2d(&tm_h, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, H, hrows, R::kKB,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MOE_OK) return rc;
  rc = encode_2d(&tm_w, w_router, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, H, std::min(npad, 256),
                 R::kKB, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MOE_OK) return rc;
  R::Params prm;
  prm.T = T;
  prm.H = H;
  prm.E = E;
  prm.k = k;
  prm.renormalize = renormalize;
  prm.do_topk = do_topk;
  prm.npad = npad;
  prm.tm = tm;
  prm.hrows = hrows;
  prm.nkb = nkb;
  prm.ns = ns;
  prm.logits = logits;
  prm.topk_idx = topk_idx;
  prm.topk_w = topk_w;
  cudaStream_t s = as_stream(stream);
  rc = keys <= 1   ? router_launch<1>(tm_h, tm_w, prm, S, tiles, smem, s)
       : keys <= 2 ? router_launch<2>(tm_h, tm_w, prm, S, tiles, smem, s)
       : keys <= 4 ? router_launch<4>(tm_h, tm_w, prm, S, tiles, smem, s)
       : keys <= 8 ? router_launch<8>(tm_h, tm_w, prm, S, tiles, smem, s)
                   : router_launch<16>(tm_h, tm_w, prm, S, tiles, smem, s);
  return rc;
}
}  // namespace

extern "C" {
int moe_router_topk(const void* h, const void* w_router, int T, int H, int E, int k,
                    int renormalize, float* logits, int32_t* topk_idx, float* topk_w,
                    void* stream) {
  const int rc = router_impl(h, w_router, T, H, E, k, renormalize, 1, logits, topk_idx, topk_w,
                             stream);
  return rc == MOE_OK ? ok() : rc;
}
}  // extern "C"

namespace {
int permute_impl(const int32_t* topk_idx, const void* x, int T, int E, int k, int H,
                 int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row, void* x_perm,
                 unsigned int* hot, void* stream) {
  MOE_CHECK(T >= 0, MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  MOE_CHECK(E >= 1 && E <= 512, MOE_ERR_UNSUPPORTED, "E=%d outside [1, 512]", E);
  MOE_CHECK(k >= 1 && k <= 16, MOE_ERR_INVALID_ARG, "k=%d outside [1, 16]", k);
  MOE_CHECK(H > 0 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "H=%d must be a positive multiple of 8", H);
  MOE_CHECK(expert_offsets != nullptr, MOE_ERR_INVALID_ARG, "null expert_offsets");
  cudaStream_t s = as_stream(stream);
  if (T == 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s));
    return ok();
  }
  MOE_CHECK(topk_idx && x && perm_token && dest_row && x_perm, MOE_ERR_INVALID_ARG,
            "null pointer");
  MOE_CHECK(aligned(x, 16) && aligned(x_perm, 16), MOE_ERR_UNSUPPORTED,
            "x and x_perm must be 16-byte aligned");
  const size_t smem = moe::permute_smem_bytes(E);
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  static std::atomic<bool> attr_set[kMaxDevices];
  if (dev >= kMaxDevices || !attr_set[dev].load()) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(moe::permute_index_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)moe::permute_smem_bytes(512)));
    if (dev < kMaxDevices) attr_set[dev].store(true);
  }
  if (T <= 2 * moe::kPermuteChunk) {  // one CTA
    MOE_CUDA_TRY(launch_pdl(moe::permute_index_kernel, dim3(1), dim3(moe::kPermuteThreads), smem,
                            s, topk_idx, T, E, k, expert_offsets, perm_token, dest_row,
                            static_cast<const int32_t*>(nullptr), hot));
  } else {
    // Split over CTAs of kPermuteChunk tokens: per-CTA expert counts first.  They
    // are kept in x_perm (nblk * E ints <= T * k * H * 2 bytes), which the row
    // gather below overwrites only after the second pass has read them.
    const int nblk = (T + moe::kPermuteChunk - 1) / moe::kPermuteChunk;
    MOE_CHECK((size_t)T * k * H * 2 >= (size_t)nblk * E * sizeof(int32_t), MOE_ERR_UNSUPPORTED,
              "x_perm too small to hold the grouping counts");
    int32_t* counts = static_cast<int32_t*>(x_perm);
    MOE_CUDA_TRY(launch_pdl(moe::permute_count_kernel, dim3(nblk), dim3(moe::kPermuteThreads),
                            (size_t)E * sizeof(int32_t), s, topk_idx, T, E, k, counts));
    MOE_CUDA_TRY(launch_pdl(moe::permute_index_kernel, dim3(nblk), dim3(moe::kPermuteThreads),
                            smem, s, topk_idx, T, E, k, expert_offsets, perm_token, dest_row,
                            static_cast<const int32_t*>(counts), hot));
  }
  const int vec = H / 8;
  const long long nvec = (long long)T * k * vec;
  const long long cap = (long long)num_sms(dev) * 8;
  const int blocks = (int)std::max(1LL, std::min(cap, (nvec + 255) / 256));
  MOE_CUDA_TRY(launch_pdl(moe::gather_rows_kernel, dim3(blocks), dim3(256), 0, s,
                          static_cast<const uint4*>(x), perm_token, expert_offsets, E, vec,
                          static_cast<uint4*>(x_perm)));
  return ok();
}
}  // namespace

extern "C" {

int moe_permute(const int32_t* topk_idx, const void* x, int T, int E, int k, int H,
                int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row, void* x_perm,
                void* stream) {
  return permute_impl(topk_idx, x, T, E, k, H, expert_offsets, perm_token, dest_row, x_perm,
                      nullptr, stream);
}

int moe_ffn_workspace_bytes(moe_layer_t L, int rows, size_t* bytes) {
  MOE_CHECK(L != nullptr && bytes != nullptr, MOE_ERR_INVALID_ARG, "null argument");
  MOE_CHECK(rows >= 0, MOE_ERR_INVALID_ARG, "rows=%d < 0", rows);
  const size_t h = ((size_t)rows * L->I * 2 + 255) / 256 * 256;
  *bytes = h + kFfnCounterBytes;  // h [rows][I] bf16, then the scheduler's counters
  return ok();
}

namespace {
int grouped_ffn_impl(moe_layer_t L, const void* x_perm, const int32_t* expert_offsets, int rows,
                     void* y_perm, void* workspace, size_t workspace_bytes, void* stream,
                     bool zero_counters);
}

int moe_grouped_ffn_mixed(moe_layer_t L, const void* x_perm, const int32_t* expert_offsets,
                          int rows, void* y_perm, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return grouped_ffn_impl(L, x_perm, expert_offsets, rows, y_perm, workspace, workspace_bytes,
                          stream, true);
}

}  // extern "C"

namespace {

// The kernel's dynamic shared-memory limit is a per-device function attribute;
// it is set once per device.
int set_ffn_attributes(int dev) {
  static std::atomic<bool> done[kMaxDevices];
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && done[dev].load()) return MOE_OK;
  MOE_CUDA_TRY(cudaFuncSetAttribute(moe::ffn::grouped_ffn_kernel<true, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    moe::ffn::kSmemLimit));
  MOE_CUDA_TRY(cudaFuncSetAttribute(moe::ffn::grouped_ffn_kernel<true, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    moe::ffn::kSmemLimit));
  MOE_CUDA_TRY(cudaFuncSetAttribute(moe::ffn::grouped_ffn_kernel<false, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    moe::ffn::kSmemLimit));
  if (cached) done[dev].store(true);
  return MOE_OK;
}

// Every host-side check of the grouped FFN, so that moe_layer_forward can run
// them before it enqueues anything.
int ffn_check(moe_layer_t L, const void* x_perm, const int32_t* expert_offsets, int rows,
              const void* y_perm, const void* workspace, size_t workspace_bytes) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(rows >= 0, MOE_ERR_INVALID_ARG, "rows=%d < 0", rows);
  if (rows == 0) return MOE_OK;
  MOE_CHECK(x_perm && expert_offsets && y_perm && workspace, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(aligned(x_perm, 16) && aligned(y_perm, 16), MOE_ERR_UNSUPPORTED,
            "x_perm and y_perm must be 16-byte aligned");
  MOE_CHECK(aligned(workspace, 256), MOE_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
  size_t need = 0;
  moe_ffn_workspace_bytes(L, rows, &need);
  MOE_CHECK(workspace_bytes >= need, MOE_ERR_INVALID_ARG, "workspace %zu B < %zu B needed",
            workspace_bytes, need);
  for (int e = 0; e < L->E; ++e)
    MOE_CHECK(L->prec[e] >= 0, MOE_ERR_NOT_MATERIALIZED, "expert %d has no weights", e);
  return MOE_OK;
}

// Launch of route_permute_gather_kernel for moe_layer_forward (T <= 128).
int route_permute_gather_small(moe_layer_t L, const float* logits, const void* x, int T,
                               int renormalize, int32_t* topk_idx, float* topk_w,
                               int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row,
                               void* x_perm, void* workspace, size_t workspace_bytes,
                               void* stream) {
  const int E = L->E, k = L->k, H = L->H;
  MOE_CHECK(logits && x && topk_idx && topk_w && expert_offsets && perm_token && dest_row &&
                x_perm,
            MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(aligned(x, 16) && aligned(x_perm, 16), MOE_ERR_UNSUPPORTED,
            "x and x_perm must be 16-byte aligned");
  size_t need = 0;
  moe_ffn_workspace_bytes(L, T * k, &need);
  MOE_CHECK(workspace != nullptr && workspace_bytes >= need, MOE_ERR_INVALID_ARG,
            "workspace %zu B < %zu B needed", workspace_bytes, need);
  int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + need - kFfnCounterBytes);
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  const int pairs = T * k;
  const int grid = std::max(1, std::min(2 * num_sms(dev), (pairs + 3) / 4));
  const size_t smem = moe::front_smem_bytes(T, k, E);
  const int keys = (E + 31) / 32;
  auto kern = keys <= 1 ? moe::route_permute_gather_kernel<1>
            : keys <= 2 ? moe::route_permute_gather_kernel<2>
            : keys <= 4 ? moe::route_permute_gather_kernel<4>
            : keys <= 8 ? moe::route_permute_gather_kernel<8>
                        : moe::route_permute_gather_kernel<16>;
  MOE_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(moe::kFrontThreads), smem, as_stream(stream),
                          logits, static_cast<const uint4*>(x), T, E, k, renormalize, H / 8,
                          topk_idx, topk_w, expert_offsets, perm_token, dest_row,
                          static_cast<uint4*>(x_perm), counters,
                          (int)(ffn_counter_bytes(E) / sizeof(int)), L->hot));
  return ok();
}

// Whether a launch of this layer can contain CUDA-core units: its shape allows
// them and some expert's base precision (a forward sees that version or a BF16
// one) spans at least kFmaMinStages stages in one of its projections.  Only
// then does the launch take the kernel instance with the CUDA-core path.
bool fma_possible(const moe_layer* L) {
  if (!fma_capable(L->H, L->I)) return false;
  for (int q : L->prec) {
    if (q != MOE_INT8 && q != MOE_INT4) continue;
    const int step = q == MOE_INT4 ? 256 : 128;
    if (L->H / step >= moe::ffn::kFmaMinStages || L->I / step >= moe::ffn::kFmaMinStages)
      return true;
  }
  return false;
}

// zero_counters = false: the caller has already zeroed the scheduler counters
// on the stream (moe_layer_forward does so first, so that no memset node sits
// between the layer's kernels).
int grouped_ffn_impl(moe_layer_t L, const void* x_perm, const int32_t* expert_offsets, int rows,
                     void* y_perm, void* workspace, size_t workspace_bytes, void* stream,
                     bool zero_counters) {
  using namespace moe::ffn;
  int rc = ffn_check(L, x_perm, expert_offsets, rows, y_perm, workspace, workspace_bytes);
  if (rc != MOE_OK || rows == 0) return rc;
  size_t need = 0;
  moe_ffn_workspace_bytes(L, rows, &need);

  cudaStream_t s = as_stream(stream);
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  const int grid = num_sms(dev);
  MOE_CHECK(grid > 0, MOE_ERR_CUDA, "cannot query the SM count");

  auto* h = static_cast<__nv_bfloat16*>(workspace);
  int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + need - kFfnCounterBytes);
  if (zero_counters) MOE_CUDA_TRY(cudaMemsetAsync(counters, 0, ffn_counter_bytes(L->E), s));

  // Every expert holds at most T = rows / k rows.  Small groups (decode) use the
  // weights-as-M orientation with a deep pipeline sized for the largest group.
  const int T = (rows + L->k - 1) / L->k;
  const bool swap = T <= 128;
  const int xrows = swap ? std::max(16, (std::min(T, 128) + 15) / 16 * 16) : 128;
  const int xbox = xrows;  // one X copy per stage
  const int nq = 4;
  // TMEM (512 columns): swap mode holds two accumulators of acc_stride columns
  // (a power of two >= the token tile), tile mode two of 256 columns.
  int acc_stride = 256;
  if (swap) {
    acc_stride = 16;
    while (acc_stride < xrows) acc_stride *= 2;
  }
  int ns = kMaxNS;
  while (ns > 2 && (int)smem_map(swap, ns, nq, xrows, L->E).total > kSmemLimit) --ns;
  const int smem = (int)smem_map(swap, ns, nq, xrows, L->E).total;
  MOE_CHECK(smem <= kSmemLimit, MOE_ERR_UNSUPPORTED, "shared memory plan does not fit");

  CUtensorMap tm_x, tm_h, tm_xf, tm_hf;
  rc = encode_2d(&tm_x, x_perm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, L->H, xbox, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MOE_OK) return rc;
  rc = encode_2d(&tm_h, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, L->I, xbox, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MOE_OK) return rc;
  // CUDA-core units (swap mode): X rows of a tile in 128-element boxes, unswizzled
  const int fma_rows = swap && fma_possible(L) ? kFmaRows : 0;
  memset(&tm_xf, 0, sizeof tm_xf);
  memset(&tm_hf, 0, sizeof tm_hf);
  if (fma_rows > 0) {
    rc = encode_2d(&tm_xf, x_perm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, L->H, kFmaRows, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != MOE_OK) return rc;
    rc = encode_2d(&tm_hf, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, L->I, kFmaRows, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != MOE_OK) return rc;
  }

  Params prm{L->d_descs, L->d_prec, expert_offsets, h, static_cast<__nv_bfloat16*>(y_perm),
             counters, counters + 16, counters + 16 + L->E, rows, L->E, L->H, L->I,
             swap ? L->I / 64 : L->I / 128, swap ? L->H / 128 : (L->H + 255) / 256,
             xbox, xrows, ns, nq, acc_stride, fma_rows};

  rc = set_ffn_attributes(dev);
  if (rc != MOE_OK) return rc;
  if (swap && fma_rows > 0)
    MOE_CUDA_TRY(launch_pdl(grouped_ffn_kernel<true, true>, dim3(grid), dim3(kThreads), smem, s,
                            tm_x, tm_h, tm_xf, tm_hf, prm));
  else if (swap)
    MOE_CUDA_TRY(launch_pdl(grouped_ffn_kernel<true, false>, dim3(grid), dim3(kThreads), smem, s,
                            tm_x, tm_h, tm_xf, tm_hf, prm));
  else
    MOE_CUDA_TRY(launch_pdl(grouped_ffn_kernel<false, false>, dim3(grid), dim3(kThreads), smem,
                            s, tm_x, tm_h, tm_xf, tm_hf, prm));
  return ok();
}
}  // namespace

// ------------------------------------------------- allocation-free FFN entry --
// Scratch for moe_grouped_ffn_mixed_noalloc: h and the scheduler counters live
// in this file-scope device array instead of a caller workspace.  Every GPU that
// loads the library holds it until the process exits.  In host code the name
// g_ffn_scratch is only a host-side stand-in, so the device address is looked up
// with cudaGetSymbolAddress, once per device, with that device current.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
__device__ __align__(256) uint8_t g_ffn_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CHECK(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_ffn_scratch);
    MOE_CHECK(e == cudaSuccess && ptr != nullptr, MOE_ERR_CUDA,
              "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}
}  // namespace

extern "C" {

int moe_grouped_ffn_mixed_noalloc(moe_layer_t L, const void* x_perm, const int32_t* expert_offsets,
                                  int rows, void* y_perm, void* stream) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(rows >= 0, MOE_ERR_INVALID_ARG, "rows=%d < 0", rows);
  if (rows == 0) return ok();
  size_t need = 0;
  moe_ffn_workspace_bytes(L, rows, &need);
  MOE_CHECK(need <= kNoAllocScratchBytes, MOE_ERR_UNSUPPORTED,
            "rows=%d needs %zu B of scratch; the built-in scratch holds %zu B "
            "(rows * I * 2 + %zu); use moe_grouped_ffn_mixed with a workspace instead",
            rows, need, kNoAllocScratchBytes, kFfnCounterBytes);
  void* scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc != MOE_OK) return rc;
  // The counters at the end of the scratch are zeroed on the stream by the call.
  return grouped_ffn_impl(L, x_perm, expert_offsets, rows, y_perm, scratch, need, stream, true);
}

int moe_ffn_noalloc_max_bytes(size_t* bytes) {
  MOE_CHECK(bytes != nullptr, MOE_ERR_INVALID_ARG, "bytes is null");
  *bytes = kNoAllocScratchBytes;
  return ok();
}

int moe_ffn_noalloc_reset(void) {
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CHECK(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  g_scratch_addr[dev] = nullptr;
  return ok();
}

int moe_combine(const void* y_perm, const int32_t* dest_row, const float* topk_w, int T, int k,
                int H, void* out, void* stream) {
  MOE_CHECK(T >= 0, MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  MOE_CHECK(k >= 1 && k <= 16, MOE_ERR_INVALID_ARG, "k=%d outside [1, 16]", k);
  MOE_CHECK(H > 0 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "H=%d must be a positive multiple of 8", H);
  if (T == 0) return ok();
  MOE_CHECK(y_perm && dest_row && topk_w && out, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(aligned(y_perm, 16) && aligned(out, 16), MOE_ERR_UNSUPPORTED,
            "y_perm and out must be 16-byte aligned");
  const int vec = H / 8;
  // decode-sized batches: 64-thread blocks, so a token's row is spread over
  // more SMs and more of its loads are in flight at once
  const int bmax = T <= 128 ? 64 : 256;
  const dim3 block(std::min(bmax, ((vec + 31) / 32) * 32));
  const dim3 grid(T, (vec + block.x - 1) / block.x);
  MOE_CUDA_TRY(launch_pdl(moe::combine_kernel, grid, block, 0, as_stream(stream),
                          static_cast<const uint4*>(y_perm), dest_row, topk_w, k, vec, T * k,
                          static_cast<uint4*>(out)));
  return ok();
}

}  // extern "C"

namespace {
// moe_layer_forward and moe_layer_forward_hidden.  w_router == NULL: the
// logits are an input; otherwise they are computed here (z = W_r x) into
// `logits`, and for T > 128 the router kernel also takes the top-k.
int layer_forward_impl(moe_layer_t L, float* logits, const void* x, const void* w_router, int T,
                       int renormalize, int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                       int32_t* perm_token, int32_t* dest_row, void* x_perm, void* y_perm,
                       void* workspace, size_t workspace_bytes, void* out, void* stream) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(T >= 0, MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0) {  // as the separate calls: no rows, every expert empty
    MOE_CHECK(expert_offsets != nullptr, MOE_ERR_INVALID_ARG, "null expert_offsets");
    MOE_CUDA_TRY(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (L->E + 1),
                                 as_stream(stream)));
    return ok();
  }
  // Every check of every step first, so that a call that fails has enqueued
  // nothing and written no output.
  int rc = ffn_check(L, x_perm, expert_offsets, T * L->k, y_perm, workspace, workspace_bytes);
  if (rc != MOE_OK) return rc;
  MOE_CHECK(logits && x && topk_idx && topk_w && perm_token && dest_row && out,
            MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(aligned(x, 16) && aligned(out, 16), MOE_ERR_UNSUPPORTED,
            "x and out must be 16-byte aligned");
  if (w_router != nullptr) {
    rc = router_check(x, w_router, T, L->H, L->E, L->k, 1, logits, topk_idx, topk_w);
    if (rc != MOE_OK) return rc;
  }
  if (T <= moe::kFrontMaxTokens) {
    // Small batch: routing, grouping and the row gather in one launch, which
    // also zeroes the FFN's scheduler counters (after the router's logits).
    if (w_router != nullptr) {
      rc = router_impl(x, w_router, T, L->H, L->E, L->k, renormalize, 0, logits, nullptr,
                       nullptr, stream);
      if (rc != MOE_OK) return rc;
    }
    rc = route_permute_gather_small(L, logits, x, T, renormalize, topk_idx, topk_w,
                                    expert_offsets, perm_token, dest_row, x_perm, workspace,
                                    workspace_bytes, stream);
    if (rc != MOE_OK) return rc;
  } else {
    // the FFN's scheduler counters, zeroed ahead of the layer's kernels
    size_t need = 0;
    moe_ffn_workspace_bytes(L, T * L->k, &need);
    MOE_CUDA_TRY(cudaMemsetAsync(static_cast<uint8_t*>(workspace) + need - kFfnCounterBytes, 0,
                                 ffn_counter_bytes(L->E), as_stream(stream)));
    if (w_router != nullptr)
      rc = router_impl(x, w_router, T, L->H, L->E, L->k, renormalize, 1, logits, topk_idx, topk_w,
                       stream);
    else
      rc = moe_route_topk(logits, T, L->E, L->k, renormalize, topk_idx, topk_w, stream);
    if (rc != MOE_OK) return rc;
    rc = permute_impl(topk_idx, x, T, L->E, L->k, L->H, expert_offsets, perm_token, dest_row,
                      x_perm, L->hot, stream);
    if (rc != MOE_OK) return rc;
  }
  rc = grouped_ffn_impl(L, x_perm, expert_offsets, T * L->k, y_perm, workspace, workspace_bytes,
                        stream, false);
  if (rc != MOE_OK) return rc;
  return moe_combine(y_perm, dest_row, topk_w, T, L->k, L->H, out, stream);
}
}  // namespace

extern "C" {
int moe_layer_forward(moe_layer_t L, const float* logits, const void* x, int T, int renormalize,
                      int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                      int32_t* perm_token, int32_t* dest_row, void* x_perm, void* y_perm,
                      void* workspace, size_t workspace_bytes, void* out, void* stream) {
  return layer_forward_impl(L, const_cast<float*>(logits), x, nullptr, T, renormalize, topk_idx,
                            topk_w, expert_offsets, perm_token, dest_row, x_perm, y_perm,
                            workspace, workspace_bytes, out, stream);
}

int moe_layer_forward_hidden(moe_layer_t L, const void* x, const void* w_router, int T,
                             int renormalize, float* logits, int32_t* topk_idx, float* topk_w,
                             int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row,
                             void* x_perm, void* y_perm, void* workspace, size_t workspace_bytes,
                             void* out, void* stream) {
  MOE_CHECK(w_router != nullptr || T == 0, MOE_ERR_INVALID_ARG, "w_router is null");
  return layer_forward_impl(L, logits, x, w_router, T, renormalize, topk_idx, topk_w,
                            expert_offsets, perm_token, dest_row, x_perm, y_perm, workspace,
                            workspace_bytes, out, stream);
}

int moe_quantize_weights(const void* w_bf16, int rows, int K, moe_precision_t precision,
                         void* q_out, void* scales, void* stream) {
  const int prec = (int)precision;
  MOE_CHECK(prec == MOE_INT8 || prec == MOE_INT4, MOE_ERR_INVALID_ARG,
            "quantiser precision must be INT8 or INT4");
  MOE_CHECK(rows >= 0 && K > 0 && K % 128 == 0, MOE_ERR_UNSUPPORTED,
            "rows=%d, K=%d (K must be a positive multiple of 128)", rows, K);
  if (rows == 0) return ok();
  MOE_CHECK(w_bf16 && q_out && scales, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CHECK(aligned(w_bf16, 8) && aligned(q_out, 4) && aligned(scales, 2), MOE_ERR_UNSUPPORTED,
            "misaligned buffer");
  const long long warps = (long long)rows * (K / 128);
  const long long blocks = (warps * 32 + 255) / 256;
  MOE_CHECK(blocks < (1LL << 31), MOE_ERR_UNSUPPORTED, "matrix too large");
  moe::quantize_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const uint16_t*>(w_bf16), rows, K, prec, static_cast<uint8_t*>(q_out),
      static_cast<uint16_t*>(scales));
  MOE_CUDA_TRY(cudaGetLastError());
  return ok();
}

int moe_layer_set_hotness_counter(moe_layer_t L, unsigned int* counts) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(counts == nullptr || aligned(counts, 4), MOE_ERR_UNSUPPORTED, "misaligned counts");
  L->hot = counts;
  return ok();
}

int moe_hot_set_size(moe_layer_t L, size_t budget_bytes, moe_precision_t low, int* n_hot) {
  MOE_CHECK(L != nullptr && n_hot != nullptr, MOE_ERR_INVALID_ARG, "null argument");
  MOE_CHECK(low == MOE_INT8 || low == MOE_INT4, MOE_ERR_INVALID_ARG,
            "the precision experts are promoted from must be INT8 or INT4");
  const size_t P = (size_t)3 * L->H * L->I;
  const size_t bf16 = 2 * P, q = (low == MOE_INT4 ? P / 2 : P) + P / 64;  // weights + fp16 scales
  const size_t n = budget_bytes / (bf16 - q);
  *n_hot = (int)std::min<size_t>(n, (size_t)L->E);
  return ok();
}

int moe_select_hot_experts(unsigned int* counts, int E, int n_hot, int zero_counts,
                           int32_t* hot_ids, void* stream) {
  MOE_CHECK(E >= 1 && E <= moe::kSelectThreads, MOE_ERR_UNSUPPORTED, "E=%d outside [1, 512]", E);
  MOE_CHECK(n_hot >= 0 && n_hot <= E, MOE_ERR_INVALID_ARG, "n_hot=%d outside [0, E]", n_hot);
  MOE_CHECK(counts != nullptr && (hot_ids != nullptr || n_hot == 0), MOE_ERR_INVALID_ARG,
            "null pointer");
  MOE_CUDA_TRY(launch_pdl(moe::select_hot_kernel, dim3(1), dim3(moe::kSelectThreads), 0,
                          as_stream(stream), counts, E, n_hot, zero_counts, hot_ids));
  return ok();
}

int moe_layer_set_bf16_slots(moe_layer_t L, int n_slots, const moe_expert_weights* slots) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(n_slots >= 0 && n_slots <= 4 * L->E, MOE_ERR_INVALID_ARG, "n_slots=%d", n_slots);
  MOE_CHECK(n_slots == 0 || slots != nullptr, MOE_ERR_INVALID_ARG, "null slots");
  std::vector<moe::ffn::ExpertDesc> h((size_t)n_slots);
  for (int i = 0; i < n_slots; ++i) {
    MOE_CHECK(slots[i].w13 != nullptr && slots[i].w2 != nullptr, MOE_ERR_INVALID_ARG,
              "null weight pointer in slot %d", i);
    MOE_CHECK(aligned(slots[i].w13, 16) && aligned(slots[i].w2, 16), MOE_ERR_UNSUPPORTED,
              "slot buffers must be 16-byte aligned");
    memset(&h[i], 0, sizeof h[i]);
    const int rc = encode_weights(&h[i], &slots[i], MOE_BF16, L->H, L->I);
    if (rc != MOE_OK) return rc;
    h[i].prec = MOE_BF16;
  }
  cudaDeviceSynchronize();  // no forward may still read the slots being replaced
  if (L->d_slots != nullptr) cudaFree(L->d_slots);
  L->d_slots = nullptr;
  L->n_slots = 0;
  if (n_slots > 0) {
    MOE_CUDA_TRY(cudaMalloc(&L->d_slots, sizeof(moe::ffn::ExpertDesc) * n_slots));
    MOE_CUDA_TRY(cudaMemcpy(L->d_slots, h.data(), sizeof(moe::ffn::ExpertDesc) * n_slots,
                            cudaMemcpyHostToDevice));
  }
  L->n_slots = n_slots;
  return ok();
}

int moe_apply_hot_set(moe_layer_t L, const int32_t* hot_ids, int n_hot, int slot_base,
                      void* stream) {
  MOE_CHECK(L != nullptr, MOE_ERR_INVALID_ARG, "layer is null");
  MOE_CHECK(n_hot >= 0 && n_hot <= L->E, MOE_ERR_INVALID_ARG, "n_hot=%d outside [0, E]", n_hot);
  MOE_CHECK(slot_base >= 0 && slot_base + n_hot <= L->n_slots, MOE_ERR_INVALID_ARG,
            "slots [%d, %d) outside the %d registered slots", slot_base, slot_base + n_hot,
            L->n_slots);
  MOE_CHECK(n_hot == 0 || hot_ids != nullptr, MOE_ERR_INVALID_ARG, "null hot_ids");
  for (int e = 0; e < L->E; ++e)
    MOE_CHECK(L->prec[e] >= 0, MOE_ERR_NOT_MATERIALIZED, "expert %d has no weights", e);
  moe::ffn::apply_hot_set_kernel<<<L->E, 64, 0, as_stream(stream)>>>(
      L->d_descs, L->d_prec, L->d_base, L->d_slots, hot_ids, n_hot, slot_base);
  MOE_CUDA_TRY(cudaGetLastError());
  return ok();
}

int moe_get_device_status(unsigned int* status) {
  MOE_CHECK(status != nullptr, MOE_ERR_INVALID_ARG, "status is null");
  MOE_CUDA_TRY(cudaDeviceSynchronize());
  unsigned int v = 0, zero = 0;
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(&v, moe::g_status, sizeof v));
  MOE_CUDA_TRY(cudaMemcpyToSymbol(moe::g_status, &zero, sizeof zero));
  *status = v;
  return ok();
}

}  // extern "C"
