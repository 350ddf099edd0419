// api.cu -- the C ABI of libwise (include/wise.h): argument validation,
// TMA descriptor construction and kernel launches.  No entry point allocates
// device memory; only wise_build_schedule with nnz_out and wise_device_status
// synchronise.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "wise.h"
#include "wise_internal.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return WISE_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(WISE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace wise {
__device__ unsigned int g_status_word = 0u;
}

namespace {

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Per-device state.  The device address of a __device__ variable belongs to the
// context the module was loaded into, so it is cached together with that context's id
// (unique for the life of the process, and new after a primary-context reset) and
// looked up again when the current context differs.
struct DeviceInfo {
  bool init = false;
  unsigned long long ctx = 0;
  int sms = 0;
  unsigned int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(WISE_ERR_CUDA, "device index %d unsupported", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  unsigned long long ctx = 0;
  const bool have_ctx = wise::current_context_id(&ctx);
  if (!di.init || !have_ctx || di.ctx != ctx) {
    e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, wise::g_status_word);   // creates the context if needed
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    di.status = static_cast<unsigned int*>(p);
    di.init = wise::current_context_id(&di.ctx);   // without an id: look up on every call
  }
  *out = &di;
  return WISE_OK;
}

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
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, n, d] bf16 viewed as a 3-D tensor (d fastest); box = 64 columns x box_rows rows,
// 128-byte swizzle, zero fill outside the tensor.
int make_tmap(CUtensorMap* map, const void* base, int d, int n, int BH, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(WISE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)n};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WISE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return WISE_OK;
}

int check_shape(const wise_shape_t& s) {
  if (s.batch < 1 || s.heads < 1)
    return fail(WISE_ERR_SHAPE, "batch (%d) and heads (%d) must be >= 1", s.batch, s.heads);
  if (s.seqlen < 32 || s.seqlen % 32 != 0 || s.seqlen > 16384)
    return fail(WISE_ERR_SHAPE, "seqlen %d must be a multiple of 32 in [32, 16384]", s.seqlen);
  if (s.head_dim != 64 && s.head_dim != 96 && s.head_dim != 128)
    return fail(WISE_ERR_SHAPE, "head_dim %d unsupported (64, 96 or 128)", s.head_dim);
  const long long bh = (long long)s.batch * s.heads;
  if (bh > (1ll << 24)) return fail(WISE_ERR_SHAPE, "batch*heads %lld too large", bh);
  if (s.kv_heads < 0 || (s.kv_heads > 0 && s.heads % s.kv_heads != 0))
    return fail(WISE_ERR_SHAPE, "heads (%d) must be a multiple of kv_heads (%d)", s.heads,
                s.kv_heads);
  if (!(std::isfinite(s.scale))) return fail(WISE_ERR_ARG, "scale must be finite");
  return WISE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float softmax_scale(const wise_shape_t& s) {
  return s.scale > 0.f ? s.scale : 1.0f / std::sqrt((float)s.head_dim);
}

int launch_attn(int mode, const void* q, const void* k, const void* v, void* o,
                const wise::AttnParams& p0, const wise_shape_t& s, void* stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc) return rc;
  const int BH = s.batch * s.heads;
  const int kv = s.kv_heads > 0 ? s.kv_heads : s.heads;
  const int BHkv = s.batch * kv;
  CUtensorMap tq, tk, tv;
  if ((rc = make_tmap(&tq, q, s.head_dim, s.seqlen, BH, 128))) return rc;
  if ((rc = make_tmap(&tk, k, s.head_dim, s.seqlen, BHkv, 32))) return rc;
  if (mode != wise::kModeMass) {
    if ((rc = make_tmap(&tv, v, s.head_dim, s.seqlen, BHkv, 32))) return rc;
  } else {
    tv = tk;
  }
  wise::AttnParams p = p0;
  p.o = o;
  p.BH = BH;
  p.group = s.heads / kv;
  p.n = s.seqlen;
  p.nq = s.seqlen / 32;
  p.num_tiles = BH * ((p.nq + 3) / 4);
  p.scale_log2 = softmax_scale(s) * 1.4426950408889634f;
  p.status = di->status;
  const int grid = p.num_tiles < di->sms ? p.num_tiles : di->sms;
  const char* why = nullptr;
  cudaError_t e = wise::launch_attention(mode, s.head_dim, tq, tk, tv, p, grid,
                                         static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) {
    if (why) return fail(WISE_ERR_CUDA, "attention launch: %s", why);
    return cuda_fail(e, "attention launch");
  }
  return WISE_OK;
}

}  // namespace

namespace wise {
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// For entry points defined in other translation units of the library.
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
int record_ok() { return ok(); }
int validate_shape(const wise_shape_t& s) { return check_shape(s); }
int status_word(unsigned int** out) {
  DeviceInfo* di = nullptr;
  const int rc = device_info(&di);
  if (rc) return rc;
  *out = di->status;
  return WISE_OK;
}
}  // namespace wise

extern "C" {

int wise_full_attn_mass(const void* q, const void* k, const void* v, void* o, float* lse,
                        float* mass, void* workspace, size_t workspace_bytes, wise_shape_t shape,
                        void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !v || !o) return fail(WISE_ERR_ARG, "q, k, v and o must be non-NULL");
  if (mass && !lse) return fail(WISE_ERR_ARG, "mass requires an lse buffer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(WISE_ERR_ALIGN, "q, k, v, o must be 16-byte aligned");
  if ((lse && !aligned16(lse)) || (mass && !aligned16(mass)))
    return fail(WISE_ERR_ALIGN, "lse and mass must be 16-byte aligned");
  const bool one_pass = mass && workspace;
  if (one_pass) {
    const size_t need = wise_mass_workspace_bytes(shape);
    if (workspace_bytes < need)
      return fail(WISE_ERR_WORKSPACE, "mass workspace of %zu bytes required", need);
    if (!aligned16(workspace)) return fail(WISE_ERR_ALIGN, "workspace must be 16-byte aligned");
  }
  wise::AttnParams p{};
  p.lse = lse;
  p.blse = one_pass ? static_cast<float*>(workspace) : nullptr;
  rc = launch_attn(wise::kModeDense, q, k, v, o, p, shape, stream);
  if (rc) return rc;
  if (one_pass) {
    cudaError_t e = wise::launch_block_mass(p.blse, lse, mass, shape.batch * shape.heads,
                                            shape.seqlen, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "mass launch");
  } else if (mass) {
    wise::AttnParams pm{};
    pm.lse_in = lse;
    pm.mass = mass;
    rc = launch_attn(wise::kModeMass, q, k, v, o, pm, shape, stream);
    if (rc) return rc;
  }
  return ok();
}

int wise_window_step(const void* q, const void* k, const void* v, void* o, float* lse,
                     float* mass, uint32_t* union_bits, uint32_t* step_bits, float eta,
                     void* workspace, size_t workspace_bytes, wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !mass || !union_bits || !workspace)
    return fail(WISE_ERR_ARG, "q, k, v, o, lse, mass, union_bits and workspace must be non-NULL");
  if (!(eta > 0.f)) return fail(WISE_ERR_ARG, "eta must be > 0 (got %g)", (double)eta);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(WISE_ERR_ALIGN, "q, k, v, o must be 16-byte aligned");
  if (!aligned16(lse) || !aligned16(mass) || !aligned16(workspace))
    return fail(WISE_ERR_ALIGN, "lse, mass and workspace must be 16-byte aligned");
  const size_t need = wise_mass_workspace_bytes(shape);
  if (workspace_bytes < need)
    return fail(WISE_ERR_WORKSPACE, "mass workspace of %zu bytes required", need);
  wise::AttnParams p{};
  p.lse = lse;
  p.blse = static_cast<float*>(workspace);
  rc = launch_attn(wise::kModeDense, q, k, v, o, p, shape, stream);
  if (rc) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = wise::launch_block_mass(p.blse, lse, mass, shape.batch * shape.heads,
                                          shape.seqlen, st);
  if (e != cudaSuccess) return cuda_fail(e, "mass launch");
  e = wise::launch_select_union(mass, union_bits, step_bits, eta, shape.batch * shape.heads,
                                shape.seqlen / 32, st);
  if (e != cudaSuccess) return cuda_fail(e, "select_union launch");
  return ok();
}

size_t wise_mass_workspace_bytes(wise_shape_t shape) {
  if (check_shape(shape)) return 0;
  const size_t nq = shape.seqlen / 32;
  return (size_t)shape.batch * shape.heads * nq * shape.seqlen * sizeof(float);
}

int wise_select_union(const float* mass, uint32_t* union_bits, uint32_t* step_bits, float eta,
                      wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!mass || !union_bits) return fail(WISE_ERR_ARG, "mass and union_bits must be non-NULL");
  if (!(eta > 0.f)) return fail(WISE_ERR_ARG, "eta must be > 0 (got %g)", (double)eta);
  const int nq = shape.seqlen / 32;
  cudaError_t e = wise::launch_select_union(mass, union_bits, step_bits, eta,
                                            shape.batch * shape.heads, nq,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_union launch");
  return ok();
}

int wise_select_union_blocks(const float* mass, uint32_t* union_bits, uint32_t* step_bits,
                             float eta, int32_t block, wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!mass || !union_bits) return fail(WISE_ERR_ARG, "mass and union_bits must be non-NULL");
  if (!(eta > 0.f)) return fail(WISE_ERR_ARG, "eta must be > 0 (got %g)", (double)eta);
  if (block != 32 && block != 64 && block != 128)
    return fail(WISE_ERR_ARG, "block must be 32, 64 or 128 (got %d)", (int)block);
  if (shape.seqlen % block != 0)
    return fail(WISE_ERR_SHAPE, "seqlen %d is not a multiple of block %d", (int)shape.seqlen,
                (int)block);
  const int nq = shape.seqlen / 32;
  cudaError_t e = wise::launch_select_union_blocks(mass, union_bits, step_bits, eta, block / 32,
                                                   shape.batch * shape.heads, nq,
                                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_union_blocks launch");
  return ok();
}

static int select_control(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                          int kind, wise_shape_t shape, void* stream, const char* what) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!mass || !ref_bits || !out_bits)
    return fail(WISE_ERR_ARG, "mass, ref_bits and out_bits must be non-NULL");
  if (ref_bits == out_bits) return fail(WISE_ERR_ARG, "out_bits must not alias ref_bits");
  const int nq = shape.seqlen / 32;
  cudaError_t e = wise::launch_select_control(mass, ref_bits, out_bits, kind,
                                              shape.batch * shape.heads, nq,
                                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, what);
  return ok();
}

int wise_select_size_matched(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                             wise_shape_t shape, void* stream) {
  return select_control(mass, ref_bits, out_bits, 0, shape, stream, "select_size_matched launch");
}

int wise_select_mass_matched(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                             wise_shape_t shape, void* stream) {
  return select_control(mass, ref_bits, out_bits, 1, shape, stream, "select_mass_matched launch");
}

int wise_support_mass(const float* mass, const uint32_t* bits, float* retained,
                      wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!mass || !bits || !retained)
    return fail(WISE_ERR_ARG, "mass, bits and retained must be non-NULL");
  const int nq = shape.seqlen / 32;
  cudaError_t e = wise::launch_support_mass(mass, bits, retained, shape.batch * shape.heads, nq,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "support_mass launch");
  return ok();
}

size_t wise_schedule_workspace_bytes(wise_shape_t shape) {
  if (check_shape(shape)) return 0;
  const long long rows = (long long)shape.batch * shape.heads * (shape.seqlen / 32);
  return wise::schedule_workspace_bytes(rows);
}

int64_t wise_schedule_max_nnz(wise_shape_t shape) {
  if (check_shape(shape)) return -1;
  const long long nq = shape.seqlen / 32;
  return (long long)shape.batch * shape.heads * nq * (nq + 1) / 2;
}

int wise_build_schedule(const uint32_t* union_bits, int32_t* row_offsets, int32_t* col_idx,
                        int64_t col_capacity, int64_t* nnz_out, void* workspace,
                        size_t workspace_bytes, wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!union_bits || !row_offsets || !col_idx)
    return fail(WISE_ERR_ARG, "union_bits, row_offsets and col_idx must be non-NULL");
  if (col_capacity < 0) return fail(WISE_ERR_ARG, "col_capacity must be >= 0");
  const long long nq = shape.seqlen / 32;
  const long long rows = (long long)shape.batch * shape.heads * nq;
  const long long max_nnz = rows * (nq + 1) / 2;
  if (max_nnz > 0x7fffffffll) return fail(WISE_ERR_SHAPE, "schedule may exceed 2^31 entries");
  const size_t need = wise::schedule_workspace_bytes(rows);
  if (!workspace || workspace_bytes < need)
    return fail(WISE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
  if (!nnz_out && col_capacity < max_nnz)
    return fail(WISE_ERR_CAPACITY,
                "col_capacity %lld < worst case %lld; pass nnz_out to check the exact size",
                (long long)col_capacity, max_nnz);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = wise::launch_build_schedule(union_bits, row_offsets, col_idx, col_capacity,
                                              workspace, rows, (int)nq, st);
  if (e != cudaSuccess) return cuda_fail(e, "build_schedule launch");
  if (nnz_out) {
    int32_t nnz = 0;
    e = cudaMemcpyAsync(&nnz, row_offsets + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading nnz");
    *nnz_out = nnz;
    if (nnz > col_capacity)
      return fail(WISE_ERR_CAPACITY, "schedule has %d entries, capacity %lld", nnz,
                  (long long)col_capacity);
  }
  return ok();
}

int wise_sparse_attn(const void* q, const void* k, const void* v, void* o,
                     const int32_t* row_offsets, const int32_t* col_idx, int64_t col_count,
                     float* lse, wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !v || !o || !row_offsets || (!col_idx && col_count > 0))
    return fail(WISE_ERR_ARG, "q, k, v, o, row_offsets, col_idx must be non-NULL");
  if (col_count < 0) return fail(WISE_ERR_ARG, "col_count must be >= 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(WISE_ERR_ALIGN, "q, k, v, o must be 16-byte aligned");
  wise::AttnParams p{};
  p.lse = lse;
  p.row_offsets = row_offsets;
  p.col_idx = col_idx;
  p.col_count = col_count;
  rc = launch_attn(wise::kModeSparse, q, k, v, o, p, shape, stream);
  if (rc) return rc;
  return ok();
}

// ------------------------------------------------------------- block size 16

int wise_block_mass_b16(const void* q, const void* k, const float* lse, float* mass16,
                        wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !lse || !mass16) return fail(WISE_ERR_ARG, "q, k, lse and mass16 must be non-NULL");
  if (!aligned16(q) || !aligned16(k)) return fail(WISE_ERR_ALIGN, "q, k must be 16-byte aligned");
  wise::AttnParams pm{};
  pm.lse_in = lse;
  pm.mass = mass16;
  pm.fine16 = 1;
  rc = launch_attn(wise::kModeMass, q, k, nullptr, nullptr, pm, shape, stream);
  if (rc) return rc;
  return ok();
}

size_t wise_mass_b16_workspace_bytes(wise_shape_t shape) {
  return 2 * wise_mass_workspace_bytes(shape);
}

int wise_full_attn_mass_b16(const void* q, const void* k, const void* v, void* o, float* lse,
                            float* mass16, void* workspace, size_t workspace_bytes,
                            wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !mass16 || !workspace)
    return fail(WISE_ERR_ARG, "q, k, v, o, lse, mass16 and workspace must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(WISE_ERR_ALIGN, "q, k, v, o must be 16-byte aligned");
  if (!aligned16(lse) || !aligned16(mass16) || !aligned16(workspace))
    return fail(WISE_ERR_ALIGN, "lse, mass16 and workspace must be 16-byte aligned");
  const size_t need = wise_mass_b16_workspace_bytes(shape);
  if (workspace_bytes < need)
    return fail(WISE_ERR_WORKSPACE, "16-token mass workspace of %zu bytes required", need);
  wise::AttnParams p{};
  p.lse = lse;
  p.blse = static_cast<float*>(workspace);
  p.fine16 = 1;
  rc = launch_attn(wise::kModeDense, q, k, v, o, p, shape, stream);
  if (rc) return rc;
  cudaError_t e = wise::launch_block_mass16(p.blse, lse, mass16, shape.batch * shape.heads,
                                            shape.seqlen, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mass16 launch");
  return ok();
}

int wise_select_union_b16(const float* mass16, uint32_t* union16, uint32_t* step16, float eta,
                          wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!mass16 || !union16) return fail(WISE_ERR_ARG, "mass16 and union16 must be non-NULL");
  if (!(eta > 0.f)) return fail(WISE_ERR_ARG, "eta must be > 0 (got %g)", (double)eta);
  cudaError_t e = wise::launch_select_union(mass16, union16, step16, eta,
                                            shape.batch * shape.heads, shape.seqlen / 16,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_union_b16 launch");
  return ok();
}

static size_t b16_bits32_offset(long long rows) {
  return (wise::schedule_workspace_bytes(rows) + 255) & ~(size_t)255;
}

size_t wise_schedule_b16_workspace_bytes(wise_shape_t shape) {
  if (check_shape(shape)) return 0;
  const long long nq = shape.seqlen / 32;
  const long long rows = (long long)shape.batch * shape.heads * nq;
  return b16_bits32_offset(rows) + (size_t)rows * ((nq + 31) / 32) * sizeof(uint32_t);
}

int wise_build_schedule_b16(const uint32_t* union16, int32_t* row_offsets, int32_t* col_idx,
                            uint8_t* sub, int64_t col_capacity, int64_t* nnz_out,
                            void* workspace, size_t workspace_bytes, wise_shape_t shape,
                            void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!union16 || !row_offsets || !col_idx || !sub)
    return fail(WISE_ERR_ARG, "union16, row_offsets, col_idx and sub must be non-NULL");
  if (col_capacity < 0) return fail(WISE_ERR_ARG, "col_capacity must be >= 0");
  const long long nq = shape.seqlen / 32;
  const long long rows = (long long)shape.batch * shape.heads * nq;
  const long long max_nnz = rows * (nq + 1) / 2;
  if (max_nnz > 0x7fffffffll) return fail(WISE_ERR_SHAPE, "schedule may exceed 2^31 entries");
  const size_t need = wise_schedule_b16_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need)
    return fail(WISE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
  if (!nnz_out && col_capacity < max_nnz)
    return fail(WISE_ERR_CAPACITY,
                "col_capacity %lld < worst case %lld; pass nnz_out to check the exact size",
                (long long)col_capacity, max_nnz);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* bits32 =
      reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + b16_bits32_offset(rows));
  const int BH = shape.batch * shape.heads;
  cudaError_t e = wise::launch_fold16(union16, bits32, BH, (int)nq, st);
  if (e == cudaSuccess)
    e = wise::launch_build_schedule(bits32, row_offsets, col_idx, col_capacity, workspace, rows,
                                    (int)nq, st);
  if (e == cudaSuccess)
    e = wise::launch_sub16(union16, row_offsets, col_idx, sub, col_capacity, BH, (int)nq, st);
  if (e != cudaSuccess) return cuda_fail(e, "build_schedule_b16 launch");
  if (nnz_out) {
    int32_t nnz = 0;
    e = cudaMemcpyAsync(&nnz, row_offsets + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading nnz");
    *nnz_out = nnz;
    if (nnz > col_capacity)
      return fail(WISE_ERR_CAPACITY, "schedule has %d entries, capacity %lld", nnz,
                  (long long)col_capacity);
  }
  return ok();
}

int wise_sparse_attn_b16(const void* q, const void* k, const void* v, void* o,
                         const int32_t* row_offsets, const int32_t* col_idx, const uint8_t* sub,
                         int64_t col_count, float* lse, wise_shape_t shape, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q || !k || !v || !o || !row_offsets || ((!col_idx || !sub) && col_count > 0))
    return fail(WISE_ERR_ARG, "q, k, v, o, row_offsets, col_idx, sub must be non-NULL");
  if (col_count < 0) return fail(WISE_ERR_ARG, "col_count must be >= 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(WISE_ERR_ALIGN, "q, k, v, o must be 16-byte aligned");
  wise::AttnParams p{};
  p.lse = lse;
  p.row_offsets = row_offsets;
  p.col_idx = col_idx;
  p.sub = sub;
  p.col_count = col_count;
  rc = launch_attn(wise::kModeSparse16, q, k, v, o, p, shape, stream);
  if (rc) return rc;
  return ok();
}

int wise_device_status(uint32_t* status_out, int clear) {
  if (!status_out) return fail(WISE_ERR_ARG, "status_out must be non-NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, wise::g_status_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "reading status");
  *status_out = v;
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(wise::g_status_word, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e, "clearing status");
  }
  return ok();
}

const char* wise_last_error(void) { return g_last_error.c_str(); }

const char* wise_version(void) { return "wise-b200 0.1.0 (sm_100a)"; }

}  // extern "C"
