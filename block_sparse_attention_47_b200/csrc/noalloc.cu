// bsa_forward_noalloc: the whole device-side call (layout, permute, pool,
// top-k selection, sparse attention, unpermute) for callers that cannot
// allocate device memory themselves.
//
// The normal entry points take every intermediate buffer from the caller.
// Some callers have no way to provide them: a plugin or FFI binding that
// only receives the tensors it is handed and has no access to the host
// application's allocator, a runtime whose memory pool is fixed at start-up
// and that forbids side allocations, or a latency-bound loop in which a
// cudaMalloc, which may synchronise the device, is not acceptable.  For them
// the intermediates live in one file-scope device array of
// BSA_NOALLOC_SCRATCH_BYTES that the library owns; the caller passes only
// Q, K, V and O.
//
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the address is fetched with
// cudaGetSymbolAddress once per device, with that device current, the first
// time the entry point runs on it.
#include <mutex>

#include "bsa_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[BSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices];

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// device address of the scratch array on the current device (set-up on the
// first call per device)
bsa_status scratch_address(void** out, const char** why) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *why = cudaGetErrorString(e);
    return BSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *why = "device ordinal out of range";
    return BSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *why = cudaGetErrorString(e);
      return BSA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" bsa_status bsa_forward_noalloc(const bsa_problem* prob, const void* q_raster,
                                          const void* k_raster, const void* v_raster,
                                          int64_t stride_b, int64_t stride_n, int64_t stride_h,
                                          void* o_raster, int64_t o_stride_b, int64_t o_stride_n,
                                          int64_t o_stride_h, int32_t* dev_status, void* stream) {
  bsa_sizes s;
  bsa_status st = bsa_query_sizes(prob, &s);
  if (st != BSA_OK) return st;  // message already set by bsa_query_sizes
  // scratch carved in this order, each piece 256-byte aligned
  const size_t need = up256(s.layout_bytes) + 4 * up256(s.perm_tensor_bytes) +
                      2 * up256(s.pool_bytes) + up256(s.idx_bytes) + up256(s.cnt_bytes);
  if (need > size_t(BSA_NOALLOC_SCRATCH_BYTES)) {
    return bsa::set_error(BSA_ERR_WORKSPACE,
                          "bsa_forward_noalloc: this problem needs %zu bytes of scratch; the "
                          "library's static scratch holds %zu (BSA_NOALLOC_SCRATCH_BYTES): use "
                          "the entry points that take caller buffers",
                          need, size_t(BSA_NOALLOC_SCRATCH_BYTES));
  }
  if (!q_raster || !k_raster || !v_raster || !o_raster) {
    return bsa::set_error(BSA_ERR_INVALID_ARG, "bsa_forward_noalloc: a raster tensor pointer is NULL");
  }
  void* base = nullptr;
  const char* why = "";
  st = scratch_address(&base, &why);
  if (st != BSA_OK) return bsa::set_error(st, "bsa_forward_noalloc: scratch address: %s", why);
  char* p = static_cast<char*>(base);
  auto take = [&](size_t n) {
    void* r = p;
    p += up256(n);
    return r;
  };
  void* layout = take(s.layout_bytes);
  void* qp = take(s.perm_tensor_bytes);
  void* kp = take(s.perm_tensor_bytes);
  void* vp = take(s.perm_tensor_bytes);
  void* op = take(s.perm_tensor_bytes);
  float* q_pool = static_cast<float*>(take(s.pool_bytes));
  float* k_pool = static_cast<float*>(take(s.pool_bytes));
  int32_t* idx = static_cast<int32_t*>(take(s.idx_bytes));
  int32_t* cnt = static_cast<int32_t*>(take(s.cnt_bytes));

  // The same sequence of entry points a caller with its own buffers makes;
  // each validates its arguments and launches on `stream`.  Every byte of
  // scratch a step reads was written by an earlier step of this call, so
  // nothing has to be cleared first.
#define BSA_STEP(call)             \
  do {                             \
    bsa_status s_ = (call);        \
    if (s_ != BSA_OK) return s_;   \
  } while (0)
  BSA_STEP(bsa_layout(prob, k_raster, stride_b, stride_n, stride_h, layout, stream));
  BSA_STEP(bsa_permute_pool(prob, layout, q_raster, k_raster, v_raster, stride_b, stride_n,
                            stride_h, qp, kp, vp, q_pool, k_pool, stream));
  BSA_STEP(bsa_select_topk(prob, q_pool, k_pool, idx, cnt, stream));
  BSA_STEP(bsa_sparse_attn_fwd(prob, layout, qp, kp, vp, idx, cnt, op, dev_status, stream));
  BSA_STEP(bsa_unpermute(prob, layout, op, o_raster, o_stride_b, o_stride_n, o_stride_h, stream));
#undef BSA_STEP
  return BSA_OK;
}
