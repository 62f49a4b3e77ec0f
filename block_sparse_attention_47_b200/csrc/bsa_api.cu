// The extern "C" entry points of libbsa.so: host-side validation of every
// argument (nothing is launched on error), derived sizes, TMA tensor maps,
// and the launches on the caller's stream.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "bsa_internal.cuh"

namespace bsa {
size_t select_smem_bytes(const Geo& g);
}

namespace {
thread_local char g_last_error[512] = "";

// one NVTX range per entry point call (free unless a profiler is attached),
// so that a timeline shows which library call queued which kernels
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace
#define BSA_RANGE() NvtxRange bsa_nvtx_range_(__func__)
namespace {
}

namespace bsa {
bsa_status set_error(bsa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}
}  // namespace bsa

namespace {

using bsa::Geo;

bsa_status fail(bsa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

bsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// library-owned status word (one per device) for callers that pass
// dev_status = NULL; read and cleared by bsa_take_default_status
__device__ int32_t g_dev_status_sink;

// test hook (bsa_debug_stall_pv): attention launches (forward and backward) made by this thread
// while it is set issue no PV; other threads' launches are unaffected
thread_local int g_stall_pv = 0;

constexpr size_t kMaxSmem = 227 * 1024;

bsa_status make_geo(const bsa_problem* p, Geo* g) {
  if (!p) return fail(BSA_ERR_INVALID_ARG, "problem is NULL");
  if (p->B < 1 || p->heads < 1) return fail(BSA_ERR_SHAPE, "B and heads must be >= 1");
  if (p->head_dim != 64 && p->head_dim != 128)
    return fail(BSA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are supported", p->head_dim);
  if (p->block_mode != BSA_BLOCK_FIXED_444 && p->block_mode != BSA_BLOCK_DYNAMIC_888)
    return fail(BSA_ERR_INVALID_ARG, "block_mode %d is not a bsa_block_mode", p->block_mode);
  const int unit = p->block_mode == BSA_BLOCK_DYNAMIC_888 ? 8 : 4;
  const int max_pad = p->block_mode == BSA_BLOCK_DYNAMIC_888 ? 1 : 3;
  const int dims[3] = {p->T, p->H, p->W};
  const int valid[3] = {p->T_valid, p->H_valid, p->W_valid};
  for (int a = 0; a < 3; ++a) {
    if (dims[a] < unit || dims[a] % unit)
      return fail(BSA_ERR_SHAPE, "grid extent %d must be a positive multiple of %d", dims[a], unit);
    if (valid[a] < 1 || valid[a] > dims[a] || dims[a] - valid[a] > max_pad)
      return fail(BSA_ERR_SHAPE,
                  "valid extent %d of %d: at most %d trailing pad rows allowed so that no "
                  "block is all pad",
                  valid[a], dims[a], max_pad);
  }
  if (p->n_prefix_segments < 0 || p->n_prefix_segments > BSA_MAX_PREFIX_SEGMENTS)
    return fail(BSA_ERR_SHAPE, "n_prefix_segments %d outside 0..%d", p->n_prefix_segments,
                BSA_MAX_PREFIX_SEGMENTS);
  if (!(std::isfinite(p->softmax_scale) && p->softmax_scale > 0.f))
    return fail(BSA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (p->block_mode == BSA_BLOCK_DYNAMIC_888 && !(std::isfinite(p->dyn_tau) && p->dyn_tau >= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "dyn_tau must be finite and >= 1 in dynamic mode");

  std::memset(g, 0, sizeof(*g));
  g->B = p->B;
  g->h = p->heads;
  g->d = p->head_dim;
  g->T = p->T;
  g->H = p->H;
  g->W = p->W;
  g->Tv = p->T_valid;
  g->Hv = p->H_valid;
  g->Wv = p->W_valid;
  g->nseg = p->n_prefix_segments;
  int64_t P = 0;
  for (int i = 0; i < g->nseg; ++i) {
    if (p->prefix_len[i] < 1) return fail(BSA_ERR_SHAPE, "prefix_len[%d] must be >= 1", i);
    g->seg_len[i] = p->prefix_len[i];
    g->seg_off[i] = int(P);
    P += (int64_t(p->prefix_len[i]) + 63) / 64 * 64;
    if (P > (int64_t(1) << 28)) return fail(BSA_ERR_SHAPE, "prefix too long");
  }
  const int64_t Nv = int64_t(p->T) * p->H * p->W;
  const int64_t N = P + Nv;
  if (N > (int64_t(1) << 28)) return fail(BSA_ERR_SHAPE, "too many tokens (%lld)", (long long)N);
  if (int64_t(p->B) * p->heads * N * p->head_dim > (int64_t(1) << 40))
    return fail(BSA_ERR_SHAPE, "tensor too large");
  g->P = int(P);
  g->Nv = int(Nv);
  g->N = int(N);
  g->nbp = int(P / 64);
  g->nbv = int(Nv / 64);
  g->nb = g->nbp + g->nbv;
  if (p->keep_blocks < 1 || p->keep_blocks > g->nbv)
    return fail(BSA_ERR_SHAPE, "keep_blocks %d outside 1..%d", p->keep_blocks, g->nbv);
  g->keep = p->keep_blocks;
  g->kcap = g->nbp + g->keep;
  g->mode = p->block_mode;
  g->nreg = p->block_mode == BSA_BLOCK_DYNAMIC_888 ? (p->T / 8) * (p->H / 8) * (p->W / 8) : 0;
  g->tau = p->dyn_tau;
  g->scale = p->softmax_scale;
  g->stall_pv = 0;
  if (int64_t(p->B) * p->heads > 65535) return fail(BSA_ERR_SHAPE, "B*heads must be <= 65535");
  if (g->nb > bsa::kAttnMaxBlocks)
    return fail(BSA_ERR_UNSUPPORTED, "%d blocks per sequence; the attention kernel walks at most %d",
                g->nb, bsa::kAttnMaxBlocks);
  if (bsa::select_smem_bytes(*g) > kMaxSmem)
    return fail(BSA_ERR_UNSUPPORTED, "too many video blocks (%d) for on-chip selection", g->nbv);
  return BSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsa_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(BSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(BSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return BSA_OK;
}

// index lists and counts are read and written as single int32 words
bsa_status check_ptr4(const void* p, const char* name) {
  if (!p) return fail(BSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) & 3u)
    return fail(BSA_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);
  return BSA_OK;
}

bsa_status check_strides(const Geo& g, int64_t sb, int64_t sn, int64_t sh, const char* name) {
  // elements; every (b, n, h) row of head_dim bf16 must start 16-byte aligned
  if (sb < 0 || sn < 0 || sh < 0 || (sb % 8) || (sn % 8) || (sh % 8))
    return fail(BSA_ERR_INVALID_ARG, "%s strides must be non-negative multiples of 8 elements",
                name);
  (void)g;  // overlapping views are the caller's business; only alignment is checked
  return BSA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*heads, N, d] bf16 block-order tensor, box = 64 columns x rows x 1
bsa_status make_map(CUtensorMap* m, const Geo& g, const void* ptr, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {cuuint64_t(g.d), cuuint64_t(g.N), cuuint64_t(g.B) * g.h};
  cuuint64_t strides[2] = {cuuint64_t(g.d) * 2, cuuint64_t(g.N) * g.d * 2};
  cuuint32_t box[3] = {64, cuuint32_t(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return BSA_OK;
}

// Raster K or V [B, N, heads, d] with heads contiguous in a token row
// (stride_h == d): maps[0] covers the prefix as 64-token boxes of
// [B, N, heads*d]; maps[1 + code] covers the video grid [B, T, H, W, heads*d]
// (starting at token P) with one box per block of shape code.
bsa_status make_raster_maps(CUtensorMap* maps, const Geo& g, const void* ptr, int64_t sb,
                            int64_t sn) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t row = cuuint64_t(g.h) * g.d;  // elements of one token row
  {
    cuuint64_t dims[3] = {row, cuuint64_t(g.N), cuuint64_t(g.B)};
    cuuint64_t strides[2] = {cuuint64_t(sn) * 2, cuuint64_t(sb) * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (raster prefix) failed (%d)", int(r));
  }
  void* video = static_cast<char*>(const_cast<void*>(ptr)) + int64_t(g.P) * sn * 2;
  for (int code = 0; code < 7; ++code) {
    int st, sh, sw;
    bsa::shape_sides(code, st, sh, sw);
    cuuint64_t dims[5] = {row, cuuint64_t(g.W), cuuint64_t(g.H), cuuint64_t(g.T), cuuint64_t(g.B)};
    cuuint64_t strides[4] = {cuuint64_t(sn) * 2, cuuint64_t(sn) * g.W * 2,
                             cuuint64_t(sn) * g.W * g.H * 2, cuuint64_t(sb) * 2};
    cuuint32_t box[5] = {64, cuuint32_t(sw), cuuint32_t(sh), cuuint32_t(st), 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(&maps[1 + code], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, video, dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (raster block shape %d) failed (%d)", code,
                  int(r));
    if (g.mode == BSA_BLOCK_FIXED_444) break;  // only the cube is used
  }
  return BSA_OK;
}

bsa_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(BSA_ERR_UNSUPPORTED, "device is sm_%d%d; libbsa is built for sm_100a", major,
                minor);
  return BSA_OK;
}

#define BSA_TRY(x)                 \
  do {                             \
    bsa_status _s = (x);           \
    if (_s != BSA_OK) return _s;   \
  } while (0)

// the caller's status word, or the library's own word of this device
bsa_status status_word(int32_t** status) {
  if (*status) return BSA_OK;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(status), g_dev_status_sink);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "cudaGetSymbolAddress(status sink)");
}

// raster K/V read by TMA boxes: heads contiguous within a token row
bsa_status check_raster_kv(const Geo& g, int64_t sh, const char* name) {
  if (sh != g.d)
    return fail(BSA_ERR_UNSUPPORTED,
                "%s: the raster attention path reads K and V as boxes of whole token rows and "
                "needs stride_h == head_dim (got %lld)",
                name, (long long)sh);
  return BSA_OK;
}

}  // namespace

extern "C" {

int32_t bsa_keep_count(int32_t n_blocks, double keep_ratio) {
  if (n_blocks < 1 || !std::isfinite(keep_ratio) || keep_ratio < 0.0 || keep_ratio > 1.0)
    return -1;
  double k = std::ceil(keep_ratio * double(n_blocks) - 1e-9);
  if (k < 1.0) k = 1.0;
  if (k > double(n_blocks)) k = double(n_blocks);
  return int32_t(k);
}

bsa_status bsa_query_sizes(const bsa_problem* prob, bsa_sizes* out) {
  g_last_error[0] = 0;
  BSA_RANGE();
  if (!out) return fail(BSA_ERR_INVALID_ARG, "out is NULL");
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  out->n_tokens = g.N;
  out->n_prefix_tokens = g.P;
  out->n_blocks = g.nb;
  out->n_prefix_blocks = g.nbp;
  out->n_video_blocks = g.nbv;
  out->n_regions = g.nreg;
  out->list_capacity = g.kcap;
  out->layout_bytes = bsa::layout_map(g).total;
  out->perm_tensor_bytes = size_t(g.B) * g.h * g.N * g.d * 2;
  out->raster_tensor_bytes = out->perm_tensor_bytes;
  out->pool_bytes = size_t(g.B) * g.h * g.nb * g.d * 4;
  out->idx_bytes = size_t(g.B) * g.h * g.nb * g.kcap * 4;
  out->cnt_bytes = size_t(g.B) * g.h * g.nb * 4;
  return BSA_OK;
}

bsa_status bsa_layout(const bsa_problem* prob, const void* k_raster, int64_t stride_b,
                      int64_t stride_n, int64_t stride_h, void* layout_buf, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  if (g.mode == BSA_BLOCK_DYNAMIC_888) {
    BSA_TRY(check_ptr(k_raster, "k_raster"));
    BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "k_raster"));
  }
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_layout(g, static_cast<const __nv_bfloat16*>(k_raster), stride_b,
                                     stride_n, stride_h, bsa::layout_ptrs(g, layout_buf),
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_layout launch");
}

bsa_status bsa_permute(const bsa_problem* prob, const void* layout_buf, const void* x_raster,
                       int64_t stride_b, int64_t stride_n, int64_t stride_h, void* x_perm,
                       void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(x_raster, "x_raster"));
  BSA_TRY(check_ptr(x_perm, "x_perm"));
  BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "x_raster"));
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_permute(g, bsa::layout_ptrs(g, const_cast<void*>(layout_buf)),
                                      static_cast<const __nv_bfloat16*>(x_raster), stride_b,
                                      stride_n, stride_h, static_cast<__nv_bfloat16*>(x_perm),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_permute launch");
}

bsa_status bsa_pool(const bsa_problem* prob, const void* layout_buf, const void* q_perm,
                    const void* k_perm, float* q_pool, float* k_pool, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(q_perm, "q_perm"));
  BSA_TRY(check_ptr(k_perm, "k_perm"));
  BSA_TRY(check_ptr(q_pool, "q_pool"));
  BSA_TRY(check_ptr(k_pool, "k_pool"));
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_pool(g, bsa::layout_ptrs(g, const_cast<void*>(layout_buf)),
                                   static_cast<const __nv_bfloat16*>(q_perm),
                                   static_cast<const __nv_bfloat16*>(k_perm), q_pool, k_pool,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_pool launch");
}

bsa_status bsa_permute_pool(const bsa_problem* prob, const void* layout_buf, const void* q_raster,
                            const void* k_raster, const void* v_raster, int64_t stride_b,
                            int64_t stride_n, int64_t stride_h, void* q_perm, void* k_perm,
                            void* v_perm, float* q_pool, float* k_pool, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(q_raster, "q_raster"));
  BSA_TRY(check_ptr(k_raster, "k_raster"));
  BSA_TRY(check_ptr(v_raster, "v_raster"));
  BSA_TRY(check_ptr(q_perm, "q_perm"));
  BSA_TRY(check_ptr(k_perm, "k_perm"));
  BSA_TRY(check_ptr(v_perm, "v_perm"));
  BSA_TRY(check_ptr(q_pool, "q_pool"));
  BSA_TRY(check_ptr(k_pool, "k_pool"));
  BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "q_raster"));
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_permute_pool(
      g, bsa::layout_ptrs(g, const_cast<void*>(layout_buf)),
      static_cast<const __nv_bfloat16*>(q_raster), static_cast<const __nv_bfloat16*>(k_raster),
      static_cast<const __nv_bfloat16*>(v_raster), stride_b, stride_n, stride_h,
      static_cast<__nv_bfloat16*>(q_perm), static_cast<__nv_bfloat16*>(k_perm),
      static_cast<__nv_bfloat16*>(v_perm), q_pool, k_pool, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_permute_pool launch");
}

// 2-D map over the pooled keys [B*heads*nb rows, d] fp32 for the TMA-fed
// score tiles (16 channels x 64 rows per box, 64-byte swizzle); false when
// the driver offers no encoder (the select kernel then loads the tiles itself)
static bool make_pool_map(CUtensorMap* m, const Geo& g, const float* k_pool) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(g.d), cuuint64_t(g.B) * g.h * g.nb};
  cuuint64_t strides[1] = {cuuint64_t(g.d) * 4};
  // 64-row boxes of 16 channels (64-byte rows): a chunk of pooled keys is
  // fetched by several issuing warps
  cuuint32_t box[2] = {16, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(k_pool), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bsa_status bsa_select_topk(const bsa_problem* prob, const float* q_pool, const float* k_pool,
                           int32_t* idx, int32_t* cnt, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(q_pool, "q_pool"));
  BSA_TRY(check_ptr(k_pool, "k_pool"));
  BSA_TRY(check_ptr4(idx, "idx"));
  BSA_TRY(check_ptr4(cnt, "cnt"));
  BSA_TRY(check_device());
  int32_t* status = nullptr;  // the library's word of this device
  BSA_TRY(status_word(&status));
  CUtensorMap kmap;
  const bool tma = make_pool_map(&kmap, g, k_pool);
  cudaError_t e = bsa::launch_select(g, q_pool, k_pool, nullptr, tma ? &kmap : nullptr, idx, cnt,
                                     status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_select_topk launch");
}

bsa_status bsa_select_topk_gated(const bsa_problem* prob, const float* q_pool,
                                 const float* k_pool, const float* gate, int32_t* idx,
                                 int32_t* cnt, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(q_pool, "q_pool"));
  BSA_TRY(check_ptr(k_pool, "k_pool"));
  BSA_TRY(check_ptr(gate, "gate"));
  BSA_TRY(check_ptr4(idx, "idx"));
  BSA_TRY(check_ptr4(cnt, "cnt"));
  BSA_TRY(check_device());
  int32_t* status = nullptr;  // the library's word of this device
  BSA_TRY(status_word(&status));
  CUtensorMap kmap;
  const bool tma = make_pool_map(&kmap, g, k_pool);
  cudaError_t e = bsa::launch_select(g, q_pool, k_pool, gate, tma ? &kmap : nullptr, idx, cnt,
                                     status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_select_topk_gated launch");
}

static bsa_status attention_common(const bsa_problem* prob, const void* layout_buf,
                                   const void* q_perm, const void* k_perm, const void* v_perm,
                                   const int32_t* idx, const int32_t* cnt, void* o_perm,
                                   int32_t* dev_status, bool dense, void* stream,
                                   float* lse = nullptr) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(q_perm, "q_perm"));
  BSA_TRY(check_ptr(k_perm, "k_perm"));
  BSA_TRY(check_ptr(v_perm, "v_perm"));
  BSA_TRY(check_ptr(o_perm, "o_perm"));
  if (!dense) {
    BSA_TRY(check_ptr4(idx, "idx"));
    BSA_TRY(check_ptr4(cnt, "cnt"));
  }
  if (lse) BSA_TRY(check_ptr4(lse, "lse"));
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u))
    return fail(BSA_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  BSA_TRY(check_device());
  bsa::KVMaps<false> maps;
  BSA_TRY(make_map(&maps.k, g, k_perm, 64));
  BSA_TRY(make_map(&maps.v, g, v_perm, 64));
  int32_t* status = dev_status;
  BSA_TRY(status_word(&status));
  g.stall_pv = g_stall_pv;
  const bsa::LayoutPtrs lp = bsa::layout_ptrs(g, const_cast<void*>(layout_buf));
  bsa::AttnIO io{};
  io.q = static_cast<const __nv_bfloat16*>(q_perm);
  io.o = static_cast<__nv_bfloat16*>(o_perm);
  io.perm = lp.perm;
  io.codes = lp.codes;
  io.bmask = lp.bmask;
  io.bfull = lp.bfull;
  io.idx = idx;
  io.cnt = cnt;
  io.status = status;
  io.lse = lse;
  cudaError_t e = bsa::launch_attention(g, maps, io, dense, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "attention launch");
}

bsa_status bsa_sparse_attn_fwd(const bsa_problem* prob, const void* layout_buf,
                               const void* q_perm, const void* k_perm, const void* v_perm,
                               const int32_t* idx, const int32_t* cnt, void* o_perm,
                               int32_t* dev_status, void* stream) {
  return attention_common(prob, layout_buf, q_perm, k_perm, v_perm, idx, cnt, o_perm, dev_status,
                          false, stream);
}

bsa_status bsa_sparse_attn_fwd_lse(const bsa_problem* prob, const void* layout_buf,
                                   const void* q_perm, const void* k_perm, const void* v_perm,
                                   const int32_t* idx, const int32_t* cnt, void* o_perm,
                                   float* lse, int32_t* dev_status, void* stream) {
  if (!lse) {
    g_last_error[0] = 0;
  BSA_RANGE();
    return fail(BSA_ERR_INVALID_ARG, "lse is NULL");
  }
  return attention_common(prob, layout_buf, q_perm, k_perm, v_perm, idx, cnt, o_perm, dev_status,
                          false, stream, lse);
}

bsa_status bsa_query_bwd_workspace(const bsa_problem* prob, size_t* bytes) {
  g_last_error[0] = 0;
  BSA_RANGE();
  if (!bytes) return fail(BSA_ERR_INVALID_ARG, "bytes is NULL");
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  const size_t nw = size_t(g.nb + 31) / 32;
  *bytes = bsa::align256(sizeof(float) * size_t(g.B) * g.h * g.N) +
           bsa::align256(sizeof(uint32_t) * size_t(g.B) * g.h * g.nb * nw);
  return BSA_OK;
}

bsa_status bsa_sparse_attn_bwd(const bsa_problem* prob, const void* layout_buf,
                               const void* q_perm, const void* k_perm, const void* v_perm,
                               const void* o_perm, const void* do_perm, const float* lse,
                               const int32_t* idx, const int32_t* cnt, void* dq_perm,
                               void* dk_perm, void* dv_perm, void* workspace, size_t ws_bytes,
                               int32_t* dev_status, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  const void* p16[] = {layout_buf, q_perm, k_perm, v_perm, o_perm, do_perm, dq_perm, dk_perm,
                       dv_perm, workspace};
  const char* n16[] = {"layout_buf", "q_perm", "k_perm", "v_perm", "o_perm", "do_perm",
                       "dq_perm", "dk_perm", "dv_perm", "workspace"};
  for (int i = 0; i < 10; ++i) BSA_TRY(check_ptr(p16[i], n16[i]));
  BSA_TRY(check_ptr(lse, "lse"));
  BSA_TRY(check_ptr4(idx, "idx"));
  BSA_TRY(check_ptr4(cnt, "cnt"));
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u))
    return fail(BSA_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  size_t need = 0;
  BSA_TRY(bsa_query_bwd_workspace(prob, &need));
  if (ws_bytes < need)
    return fail(BSA_ERR_WORKSPACE, "workspace of %zu bytes; the backward needs %zu", ws_bytes,
                need);
  BSA_TRY(check_device());
  g.stall_pv = g_stall_pv;
  CUtensorMap maps[4];
  BSA_TRY(make_map(&maps[0], g, k_perm, 64));
  BSA_TRY(make_map(&maps[1], g, v_perm, 64));
  BSA_TRY(make_map(&maps[2], g, q_perm, 64));
  BSA_TRY(make_map(&maps[3], g, do_perm, 64));
  int32_t* status = dev_status;
  BSA_TRY(status_word(&status));
  const bsa::LayoutPtrs lp = bsa::layout_ptrs(g, const_cast<void*>(layout_buf));
  bsa::BwdIO io{};
  io.q = static_cast<const __nv_bfloat16*>(q_perm);
  io.k = static_cast<const __nv_bfloat16*>(k_perm);
  io.v = static_cast<const __nv_bfloat16*>(v_perm);
  io.o = static_cast<const __nv_bfloat16*>(o_perm);
  io.dout = static_cast<const __nv_bfloat16*>(do_perm);
  io.lse = lse;
  io.delta = static_cast<float*>(workspace);
  io.kmask = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) +
                                         bsa::align256(sizeof(float) * size_t(g.B) * g.h * g.N));
  io.idx = idx;
  io.cnt = cnt;
  io.bmask = lp.bmask;
  io.bfull = lp.bfull;
  io.dq = static_cast<__nv_bfloat16*>(dq_perm);
  io.dk = static_cast<__nv_bfloat16*>(dk_perm);
  io.dv = static_cast<__nv_bfloat16*>(dv_perm);
  io.status = status;
  cudaError_t e = bsa::launch_attention_bwd(g, maps, io, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "backward launch");
}

bsa_status bsa_dense_attn_fwd(const bsa_problem* prob, const void* layout_buf,
                              const void* q_perm, const void* k_perm, const void* v_perm,
                              void* o_perm, int32_t* dev_status, void* stream) {
  return attention_common(prob, layout_buf, q_perm, k_perm, v_perm, nullptr, nullptr, o_perm,
                          dev_status, true, stream);
}

bsa_status bsa_unpermute(const bsa_problem* prob, const void* layout_buf, const void* o_perm,
                         void* o_raster, int64_t stride_b, int64_t stride_n, int64_t stride_h,
                         void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(o_perm, "o_perm"));
  BSA_TRY(check_ptr(o_raster, "o_raster"));
  BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "o_raster"));
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_unpermute(g, bsa::layout_ptrs(g, const_cast<void*>(layout_buf)),
                                        static_cast<const __nv_bfloat16*>(o_perm),
                                        static_cast<__nv_bfloat16*>(o_raster), stride_b,
                                        stride_n, stride_h, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_unpermute launch");
}

// ---- raster order: no permuted copies ---------------------------------------
bsa_status bsa_pool_raster(const bsa_problem* prob, const void* layout_buf, const void* q_raster,
                           const void* k_raster, int64_t stride_b, int64_t stride_n,
                           int64_t stride_h, float* q_pool, float* k_pool, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(q_raster, "q_raster"));
  BSA_TRY(check_ptr(k_raster, "k_raster"));
  BSA_TRY(check_ptr(q_pool, "q_pool"));
  BSA_TRY(check_ptr(k_pool, "k_pool"));
  BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "q_raster/k_raster"));
  BSA_TRY(check_device());
  cudaError_t e = bsa::launch_pool_raster(
      g, bsa::layout_ptrs(g, const_cast<void*>(layout_buf)),
      static_cast<const __nv_bfloat16*>(q_raster), static_cast<const __nv_bfloat16*>(k_raster),
      stride_b, stride_n, stride_h, q_pool, k_pool, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "bsa_pool_raster launch");
}

static bsa_status raster_attention(const bsa_problem* prob, const void* layout_buf,
                                   const void* q_raster, const void* k_raster,
                                   const void* v_raster, int64_t stride_b, int64_t stride_n,
                                   int64_t stride_h, const int32_t* idx, const int32_t* cnt,
                                   const int32_t* windows, void* o_raster, int64_t o_stride_b,
                                   int64_t o_stride_n, int64_t o_stride_h, int32_t* dev_status,
                                   void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  BSA_TRY(check_ptr(q_raster, "q_raster"));
  BSA_TRY(check_ptr(k_raster, "k_raster"));
  BSA_TRY(check_ptr(v_raster, "v_raster"));
  BSA_TRY(check_ptr(o_raster, "o_raster"));
  if (windows) {
    BSA_TRY(check_ptr4(windows, "windows"));
  } else {
    BSA_TRY(check_ptr4(idx, "idx"));
    BSA_TRY(check_ptr4(cnt, "cnt"));
  }
  BSA_TRY(check_strides(g, stride_b, stride_n, stride_h, "q_raster/k_raster/v_raster"));
  BSA_TRY(check_strides(g, o_stride_b, o_stride_n, o_stride_h, "o_raster"));
  BSA_TRY(check_raster_kv(g, stride_h, "k_raster/v_raster"));
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u))
    return fail(BSA_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  BSA_TRY(check_device());
  bsa::KVMaps<true> maps{};
  BSA_TRY(make_raster_maps(maps.k, g, k_raster, stride_b, stride_n));
  BSA_TRY(make_raster_maps(maps.v, g, v_raster, stride_b, stride_n));
  int32_t* status = dev_status;
  BSA_TRY(status_word(&status));
  g.stall_pv = g_stall_pv;
  const bsa::LayoutPtrs lp = bsa::layout_ptrs(g, const_cast<void*>(layout_buf));
  bsa::AttnIO io{};
  io.q = static_cast<const __nv_bfloat16*>(q_raster);
  io.qsb = stride_b;
  io.qsn = stride_n;
  io.qsh = stride_h;
  io.o = static_cast<__nv_bfloat16*>(o_raster);
  io.osb = o_stride_b;
  io.osn = o_stride_n;
  io.osh = o_stride_h;
  io.perm = lp.perm;
  io.codes = lp.codes;
  io.bmask = lp.bmask;
  io.bfull = lp.bfull;
  io.idx = idx;
  io.cnt = cnt;
  io.status = status;
  io.windows = windows;
  cudaError_t e = bsa::launch_attention_raster(g, maps, io, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "raster attention launch");
}

bsa_status bsa_sparse_attn_fwd_raster(const bsa_problem* prob, const void* layout_buf,
                                      const void* q_raster, const void* k_raster,
                                      const void* v_raster, int64_t stride_b, int64_t stride_n,
                                      int64_t stride_h, const int32_t* idx, const int32_t* cnt,
                                      void* o_raster, int64_t o_stride_b, int64_t o_stride_n,
                                      int64_t o_stride_h, int32_t* dev_status, void* stream) {
  return raster_attention(prob, layout_buf, q_raster, k_raster, v_raster, stride_b, stride_n,
                          stride_h, idx, cnt, nullptr, o_raster, o_stride_b, o_stride_n,
                          o_stride_h, dev_status, stream);
}

bsa_status bsa_window_attn_fwd_raster(const bsa_problem* prob, const void* layout_buf,
                                      const void* q_raster, const void* k_raster,
                                      const void* v_raster, int64_t stride_b, int64_t stride_n,
                                      int64_t stride_h, const int32_t* windows, void* o_raster,
                                      int64_t o_stride_b, int64_t o_stride_n, int64_t o_stride_h,
                                      int32_t* dev_status, void* stream) {
  if (!windows) {
    g_last_error[0] = 0;
  BSA_RANGE();
    return fail(BSA_ERR_INVALID_ARG, "windows is NULL");
  }
  return raster_attention(prob, layout_buf, q_raster, k_raster, v_raster, stride_b, stride_n,
                          stride_h, nullptr, nullptr, windows, o_raster, o_stride_b, o_stride_n,
                          o_stride_h, dev_status, stream);
}

// ---- whole call from host memory -------------------------------------------
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_copy_mutex;
cudaStream_t g_copy_in[kMaxDevices], g_copy_out[kMaxDevices], g_compute[kMaxDevices];

// the library's streams of the current device (uploads, downloads and a
// second compute stream), created on first use
bsa_status side_streams(cudaStream_t* in, cudaStream_t* out, cudaStream_t* cmp) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BSA_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(g_copy_mutex);
  if (!g_copy_in[dev]) {
    e = cudaStreamCreateWithFlags(&g_copy_in[dev], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&g_copy_out[dev], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&g_compute[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
  }
  *in = g_copy_in[dev];
  *out = g_copy_out[dev];
  *cmp = g_compute[dev];
  return BSA_OK;
}

// events of one call, destroyed on every exit (pending work keeps them alive)
struct EventSet {
  std::vector<cudaEvent_t> ev;
  ~EventSet() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaError_t make(size_t n) {
    ev.reserve(n);
    for (size_t i = 0; i < n; ++i) {
      cudaEvent_t e;
      cudaError_t r = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
      if (r != cudaSuccess) return r;
      ev.push_back(e);
    }
    return cudaSuccess;
  }
};

}  // namespace

bsa_status bsa_forward_host(const bsa_problem* prob, const void* q_host, const void* k_host,
                            const void* v_host, void* o_host, const bsa_device_buffers* buf,
                            int32_t heads_per_group, int32_t* dev_status, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  if (!q_host || !k_host || !v_host || !o_host)
    return fail(BSA_ERR_INVALID_ARG, "a host tensor pointer is NULL");
  if (!buf) return fail(BSA_ERR_INVALID_ARG, "buf is NULL");
  const void* dev_ptrs[] = {buf->q_raster, buf->k_raster, buf->v_raster, buf->o_raster,
                            buf->q_perm,   buf->k_perm,   buf->v_perm,   buf->o_perm,
                            buf->layout_buf, buf->q_pool, buf->k_pool,   buf->idx,
                            buf->cnt};
  const char* dev_names[] = {"q_raster", "k_raster", "v_raster", "o_raster", "q_perm",
                             "k_perm",   "v_perm",   "o_perm",   "layout_buf", "q_pool",
                             "k_pool",   "idx",      "cnt"};
  // no permuted buffers at all: the permute-free path reads the tiles
  // straight from the raster buffers
  const bool raster = !buf->q_perm && !buf->k_perm && !buf->v_perm && !buf->o_perm;
  for (int i = 0; i < 11; ++i)
    if (!(raster && i >= 4 && i < 8)) BSA_TRY(check_ptr(dev_ptrs[i], dev_names[i]));
  BSA_TRY(check_ptr4(buf->idx, "idx"));
  BSA_TRY(check_ptr4(buf->cnt, "cnt"));
  if (heads_per_group < 1 || heads_per_group > g.h || g.h % heads_per_group != 0)
    return fail(BSA_ERR_INVALID_ARG, "heads_per_group %d must divide heads (%d)", heads_per_group,
                g.h);
  BSA_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream), s_in, s_out, s_c2;
  BSA_TRY(side_streams(&s_in, &s_out, &s_c2));

  const int groups = g.h / heads_per_group;
  bsa_problem sub = *prob;
  sub.heads = heads_per_group;
  Geo gs;
  BSA_TRY(make_geo(&sub, &gs));
  // raster [B, N, heads, d]: a head group is a strided slab of every token row
  const int64_t sn = int64_t(g.h) * g.d, sb = int64_t(g.N) * sn, sh = g.d;
  const size_t pitch = size_t(sn) * 2, width = size_t(heads_per_group) * g.d * 2;
  const size_t rows = size_t(g.B) * g.N;
  const size_t perm_elems = size_t(g.B) * heads_per_group * g.N * g.d;   // per group
  const size_t pool_elems = size_t(g.B) * heads_per_group * g.nb * g.d;
  const size_t idx_elems = size_t(g.B) * heads_per_group * g.nb * g.kcap;
  const size_t cnt_elems = size_t(g.B) * heads_per_group * g.nb;
  const bool dynamic = g.mode == BSA_BLOCK_DYNAMIC_888;

  EventSet es;  // start, k, in[groups], out[groups], done, layout
  cudaError_t e = es.make(4 + 2 * size_t(groups));
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreateWithFlags");
  cudaEvent_t ev_start = es.ev[0], ev_k = es.ev[1], ev_done = es.ev[2 + 2 * groups];
  cudaEvent_t ev_layout = es.ev[3 + 2 * groups];
  auto ev_in = [&](int i) { return es.ev[2 + i]; };
  auto ev_out = [&](int i) { return es.ev[2 + groups + i]; };
  auto slab = [&](const void* base, int grp) {
    return static_cast<const char*>(base) + size_t(grp) * width;
  };
#define BSA_CUDA(call, what)                 \
  do {                                       \
    cudaError_t e_ = (call);                 \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)
  // the copy streams start after the work already queued on the caller's stream
  BSA_CUDA(cudaEventRecord(ev_start, st), "cudaEventRecord");
  BSA_CUDA(cudaStreamWaitEvent(s_in, ev_start, 0), "cudaStreamWaitEvent");
  BSA_CUDA(cudaStreamWaitEvent(s_out, ev_start, 0), "cudaStreamWaitEvent");

  // the dynamic layout looks at every head of K: copy K whole first
  if (dynamic) {
    BSA_CUDA(cudaMemcpyAsync(buf->k_raster, k_host, rows * pitch, cudaMemcpyHostToDevice, s_in),
             "cudaMemcpyAsync K");
    BSA_CUDA(cudaEventRecord(ev_k, s_in), "cudaEventRecord");
    BSA_CUDA(cudaStreamWaitEvent(st, ev_k, 0), "cudaStreamWaitEvent");
  }
  BSA_TRY(bsa_layout(prob, buf->k_raster, sb, sn, sh, buf->layout_buf, st));
  // odd groups compute on the library's second stream, so that a group's
  // first kernels fill the SMs that the previous group's last ones leave idle
  BSA_CUDA(cudaEventRecord(ev_layout, st), "cudaEventRecord");
  BSA_CUDA(cudaStreamWaitEvent(s_c2, ev_layout, 0), "cudaStreamWaitEvent");

  // uploads: every group's slabs, in order, on the input stream
  for (int i = 0; i < groups; ++i) {
    const void* hosts[3] = {q_host, k_host, v_host};
    void* devs[3] = {buf->q_raster, buf->k_raster, buf->v_raster};
    for (int t = 0; t < 3; ++t) {
      if (t == 1 && dynamic) continue;
      BSA_CUDA(cudaMemcpy2DAsync(const_cast<char*>(slab(devs[t], i)), pitch, slab(hosts[t], i),
                                 pitch, width, rows, cudaMemcpyHostToDevice, s_in),
               "cudaMemcpy2DAsync upload");
    }
    BSA_CUDA(cudaEventRecord(ev_in(i), s_in), "cudaEventRecord");
  }
  // computation of each group once its slabs have landed
  for (int i = 0; i < groups; ++i) {
    const cudaStream_t cs = (i & 1) ? s_c2 : st;
    BSA_CUDA(cudaStreamWaitEvent(cs, ev_in(i), 0), "cudaStreamWaitEvent");
    const int64_t h0 = int64_t(i) * heads_per_group * g.d;  // element offset of the slab
    auto rq = static_cast<const __nv_bfloat16*>(buf->q_raster) + h0;
    auto rk = static_cast<const __nv_bfloat16*>(buf->k_raster) + h0;
    auto rv = static_cast<const __nv_bfloat16*>(buf->v_raster) + h0;
    auto ro = static_cast<__nv_bfloat16*>(buf->o_raster) + h0;
    auto pq = static_cast<__nv_bfloat16*>(buf->q_perm) + i * perm_elems;
    auto pk = static_cast<__nv_bfloat16*>(buf->k_perm) + i * perm_elems;
    auto pv = static_cast<__nv_bfloat16*>(buf->v_perm) + i * perm_elems;
    auto po = static_cast<__nv_bfloat16*>(buf->o_perm) + i * perm_elems;
    float* qpool = buf->q_pool + i * pool_elems;
    float* kpool = buf->k_pool + i * pool_elems;
    int32_t* idx = buf->idx + i * idx_elems;
    int32_t* cnt = buf->cnt + i * cnt_elems;
    if (raster) {
      BSA_TRY(bsa_pool_raster(&sub, buf->layout_buf, rq, rk, sb, sn, sh, qpool, kpool, cs));
      BSA_TRY(bsa_select_topk(&sub, qpool, kpool, idx, cnt, cs));
      BSA_TRY(bsa_sparse_attn_fwd_raster(&sub, buf->layout_buf, rq, rk, rv, sb, sn, sh, idx, cnt,
                                         ro, sb, sn, sh, dev_status, cs));
    } else {
      BSA_TRY(bsa_permute_pool(&sub, buf->layout_buf, rq, rk, rv, sb, sn, sh, pq, pk, pv, qpool,
                               kpool, cs));
      BSA_TRY(bsa_select_topk(&sub, qpool, kpool, idx, cnt, cs));
      BSA_TRY(bsa_sparse_attn_fwd(&sub, buf->layout_buf, pq, pk, pv, idx, cnt, po, dev_status,
                                  cs));
      BSA_TRY(bsa_unpermute(&sub, buf->layout_buf, po, ro, sb, sn, sh, cs));
    }
    BSA_CUDA(cudaEventRecord(ev_out(i), cs), "cudaEventRecord");
  }
  // downloads on the output stream; the caller's stream ends with the last one
  for (int i = 0; i < groups; ++i) {
    BSA_CUDA(cudaStreamWaitEvent(s_out, ev_out(i), 0), "cudaStreamWaitEvent");
    BSA_CUDA(cudaMemcpy2DAsync(const_cast<char*>(slab(o_host, i)), pitch, slab(buf->o_raster, i),
                               pitch, width, rows, cudaMemcpyDeviceToHost, s_out),
             "cudaMemcpy2DAsync download");
  }
  BSA_CUDA(cudaEventRecord(ev_done, s_out), "cudaEventRecord");
  BSA_CUDA(cudaStreamWaitEvent(st, ev_done, 0), "cudaStreamWaitEvent");
#undef BSA_CUDA
  return BSA_OK;
}

bsa_status bsa_debug_stall_pv(int32_t enable) {
  g_last_error[0] = 0;
  BSA_RANGE();
  g_stall_pv = enable ? 1 : 0;
  return BSA_OK;
}

bsa_status bsa_take_default_status(int32_t* out, void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  if (!out) return fail(BSA_ERR_INVALID_ARG, "out is NULL");
  BSA_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  const int32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_dev_status_sink, sizeof(v), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_dev_status_sink, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "bsa_take_default_status");
  *out = v;
  return BSA_OK;
}

bsa_status bsa_layout_stats(const bsa_problem* prob, const void* layout_buf, int64_t hist7[7],
                            void* stream) {
  g_last_error[0] = 0;
  BSA_RANGE();
  Geo g;
  BSA_TRY(make_geo(prob, &g));
  BSA_TRY(check_ptr(layout_buf, "layout_buf"));
  if (!hist7) return fail(BSA_ERR_INVALID_ARG, "hist7 is NULL");
  for (int i = 0; i < 7; ++i) hist7[i] = 0;
  if (g.mode == BSA_BLOCK_FIXED_444) {
    hist7[0] = int64_t(g.B) * g.nbv;
    return BSA_OK;
  }
  BSA_TRY(check_device());
  const size_t n = size_t(g.B) * g.nreg;
  unsigned char* host = static_cast<unsigned char*>(malloc(n));
  if (!host) return fail(BSA_ERR_HOST_MEMORY, "host allocation of %zu bytes failed", n);
  const char* src = static_cast<const char*>(layout_buf) + bsa::layout_map(g).codes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host, src, n, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    free(host);
    return cuda_fail(e, "bsa_layout_stats copy");
  }
  for (size_t i = 0; i < n; ++i) hist7[host[i] < 7 ? host[i] : 0] += 8;
  free(host);
  return BSA_OK;
}

const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_SHAPE: return "BSA_ERR_SHAPE";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_HOST_MEMORY: return "BSA_ERR_HOST_MEMORY";
  }
  return "BSA_ERR_UNKNOWN";
}

const char* bsa_last_error(void) { return g_last_error; }

}  // extern "C"
