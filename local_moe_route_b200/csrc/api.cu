// api.cu -- the C ABI declared in include/strata_moe.h: host-side argument
// validation, the scratch-space layout, the device check word, and the
// order of kernel launches for each entry point.  No entry point allocates
// or frees memory, and none synchronises the host except
// strata_moe_device_status.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/strata_moe.h"
#include "common.cuh"
#include "internal.h"

namespace strata {

// Device-side check word (one per device that loads the library).
__device__ unsigned g_check_word;

unsigned* check_word();
static unsigned* check_word_ptr() { return check_word(); }

// Device address of g_check_word on the current device, looked up once per
// device and cached.
unsigned* check_word() {
  static std::mutex mu;
  static unsigned* cache[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_check_word) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned*>(p);
  }
  return cache[dev];
}

// Streaming multiprocessors of the current device, looked up once per device.
int sm_count() {
  static std::mutex mu;
  static int cache[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

CUresult encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                        uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                        CUtensorMapL2promotion promo) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

namespace {

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- validation -----------------------------------------------------------
strata_status_t check_dims(const strata_moe_dims_t& d) {
  if (d.T < 0 || d.d <= 0 || d.E <= 0 || d.k <= 0 || d.n <= 0 || d.group <= 0 || d.k > d.E)
    return STRATA_ERR_INVALID_ARG;
  if (d.d % 128 || d.n % 128) return STRATA_ERR_UNSUPPORTED;
  if (d.group != 32 && d.group != 64 && d.group != 128) return STRATA_ERR_UNSUPPORTED;
  if (d.E > 1024 || d.k > 32) return STRATA_ERR_UNSUPPORTED;
  if ((int64_t)d.T * d.k >= (int64_t(1) << 31)) return STRATA_ERR_UNSUPPORTED;
  if ((int64_t)d.T * d.d >= (int64_t(1) << 40)) return STRATA_ERR_UNSUPPORTED;
  return STRATA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

// ---- scratch layouts --------------------------------------------------------
struct Region {
  size_t off = 0, bytes = 0;
};

struct Layout {
  size_t total = 0;
  Region add(size_t bytes) {
    Region r;
    r.off = total;
    r.bytes = bytes;
    total += up256(bytes);
    return r;
  }
};

size_t route_scratch(const strata_moe_dims_t& d) {
  const int ks = router_ksplit(d.T, d.d, d.E);
  return up256((size_t)ks * d.T * d.E * sizeof(float));
}
size_t permute_scratch(const strata_moe_dims_t& d) {
  const size_t S = (size_t)d.T * d.k;
  const size_t nchunks = (S + kPermChunk - 1) / kPermChunk;
  return up256(nchunks * d.E * sizeof(int32_t));
}

struct SchedRegions {
  Region tile_prefix, tile_table, active, n_active;
};
SchedRegions add_schedule(Layout& L, const strata_moe_dims_t& d) {
  const int S = d.T * d.k;
  SchedRegions r;
  r.tile_prefix = L.add((size_t)(d.E + 1) * sizeof(int32_t));
  r.tile_table = L.add((size_t)max_tiles(S, d.E) * sizeof(int4));
  r.active = L.add((size_t)d.E * sizeof(int32_t));
  r.n_active = L.add(sizeof(int32_t));
  return r;
}
Schedule schedule_at(uint8_t* ws, const SchedRegions& r) {
  Schedule s;
  s.tile_prefix = reinterpret_cast<int32_t*>(ws + r.tile_prefix.off);
  s.tile_table = reinterpret_cast<int4*>(ws + r.tile_table.off);
  s.active = reinterpret_cast<int32_t*>(ws + r.active.off);
  s.n_active = reinterpret_cast<int32_t*>(ws + r.n_active.off);
  return s;
}
// fp16 rows of x in grouped order [T*k][d], the B operand of the tensor-core
// gate/up path (batches above the streaming threshold).
size_t x16_bytes(const strata_moe_dims_t& d) {
  return d.T > kStreamMaxTokens ? (size_t)d.T * d.k * d.d * 2 : 0;
}
size_t gemm_scratch(const strata_moe_dims_t& d) {
  Layout L;
  add_schedule(L, d);
  L.add(x16_bytes(d));
  return L.total;
}

struct ForwardLayout {
  Region ids, w, partial, counts, offsets, sorted_token, slot_row, hist, x16, h, rows, fused;
  SchedRegions sched;
  size_t total;
};
ForwardLayout forward_layout(const strata_moe_dims_t& d) {
  const size_t S = (size_t)d.T * d.k;
  Layout L;
  ForwardLayout f;
  f.ids = L.add(S * sizeof(int32_t));
  f.w = L.add(S * sizeof(float));
  f.partial = L.add(route_scratch(d));
  f.counts = L.add((size_t)d.E * sizeof(int32_t));
  f.offsets = L.add((size_t)(d.E + 1) * sizeof(int32_t));
  f.sorted_token = L.add(S * sizeof(int32_t));
  f.slot_row = L.add(S * sizeof(int32_t));
  f.hist = L.add(permute_scratch(d));
  f.sched = add_schedule(L, d);
  f.x16 = L.add(x16_bytes(d));
  f.h = L.add(S * (size_t)d.n * 2);
  f.rows = L.add(S * (size_t)d.d * 2);
  f.fused = L.add(decode_fused_fits(d.T, d.d, d.E, d.k, d.n, d.group)
                      ? decode_fused_scratch(d.T, d.d, d.E, d.k, d.n)
                      : 0);
  f.total = L.total;
  return f;
}

strata_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? STRATA_OK : STRATA_ERR_CUDA; }

// ---- the steps, shared by the standalone entry points and forward ---------
strata_status_t do_route(const uint16_t* x, const uint16_t* w_router, const float* bias,
                         const strata_moe_dims_t& d, int32_t* ids, float* w, float* logits_out,
                         float* partial, unsigned* err, cudaStream_t s) {
  const int ks = router_ksplit(d.T, d.d, d.E);
  cudaError_t e;
  if (router_uses_tc(d.T, d.d, d.E))
    e = launch_router_logits_tc(x, w_router, d.T, d.d, d.E, partial, err, s);
  else
    e = launch_router_logits_simt(x, w_router, d.T, d.d, d.E, ks, partial, s);
  if (e != cudaSuccess) return STRATA_ERR_CUDA;
  // either path leaves the logits in split 0 of `partial`
  return cuda_status(launch_topk_softmax(partial, 1, bias, d.T, d.E, d.k, ids, w, logits_out, s));
}

strata_status_t do_gemm(int op, const uint16_t* a, const int32_t* sorted_token,
                        const int32_t* offsets, strata_q4_t w0, strata_q4_t w1,
                        const float* row_scale, const strata_moe_dims_t& d, uint16_t* out,
                        const Schedule& sch, uint16_t* x16, unsigned* err, cudaStream_t s,
                        bool h_interleaved = false) {
  GemmProblem p;
  p.op = op;
  p.a = a;
  p.a16 = x16;
  p.sorted_token = sorted_token;
  p.offsets = offsets;
  p.q0 = w0.q;
  p.s0 = w0.s;
  p.q1 = w1.q;
  p.s1 = w1.s;
  p.row_scale = row_scale;
  p.out = out;
  p.T = d.T;
  p.S = d.T * d.k;
  p.E = d.E;
  p.K = op == 0 ? d.d : d.n;
  p.N = op == 0 ? d.n : d.d;
  p.G = d.group;
  p.err = err;
  p.h_interleaved = h_interleaved;
  cudaError_t e;
  if (d.T > kStreamMaxTokens) {
    e = launch_gemm_tc(p, sch, s);
  } else {
    e = launch_gemm_decode(p, sch, s);
    if (e == cudaErrorNotSupported) e = launch_gemm_stream(p, sch, s);
  }
  return cuda_status(e);
}

}  // namespace
}  // namespace strata

using namespace strata;

extern "C" {

size_t strata_moe_workspace_bytes(strata_moe_dims_t dims) {
  if (check_dims(dims) != STRATA_OK) return 0;
  return forward_layout(dims).total;
}

const char* strata_status_string(strata_status_t status) {
  switch (status) {
    case STRATA_OK: return "ok";
    case STRATA_ERR_INVALID_ARG: return "invalid argument";
    case STRATA_ERR_UNSUPPORTED: return "unsupported shape";
    case STRATA_ERR_WORKSPACE: return "workspace missing or too small";
    case STRATA_ERR_CUDA: return "CUDA error";
    case STRATA_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

strata_status_t strata_moe_route(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                 strata_moe_dims_t dims, int32_t* topk_ids, float* topk_w,
                                 float* logits_out, void* ws, size_t ws_bytes,
                                 strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (dims.T == 0) return STRATA_OK;   // empty batch: nothing to read or write
  if (!ok_ptr(x) || !ok_ptr(w_router) || !ok_opt(bias) || !ok_ptr(topk_ids) || !ok_ptr(topk_w) ||
      !ok_opt(logits_out))
    return STRATA_ERR_INVALID_ARG;
  if (!ok_ptr(ws) || ws_bytes < route_scratch(dims)) return STRATA_ERR_WORKSPACE;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  return do_route(x, w_router, bias, dims, topk_ids, topk_w, logits_out,
                  static_cast<float*>(ws), err, reinterpret_cast<cudaStream_t>(stream));
}

strata_status_t strata_moe_permute(const int32_t* topk_ids, strata_moe_dims_t dims,
                                   int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                                   int32_t* slot_row, void* ws, size_t ws_bytes,
                                   strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return STRATA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dims.T == 0) {
    // empty batch: every count and offset is zero
    if (cudaMemsetAsync(counts, 0, (size_t)dims.E * 4, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (size_t)(dims.E + 1) * 4, s) != cudaSuccess)
      return STRATA_ERR_CUDA;
    return STRATA_OK;
  }
  if (!ok_ptr(topk_ids) || !ok_ptr(sorted_token) || !ok_ptr(slot_row)) return STRATA_ERR_INVALID_ARG;
  if (!ok_ptr(ws) || ws_bytes < permute_scratch(dims)) return STRATA_ERR_WORKSPACE;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  return cuda_status(launch_permute(topk_ids, dims.T, dims.k, dims.E, counts, offsets,
                                    sorted_token, slot_row, static_cast<int32_t*>(ws), err, s));
}

// Fixed scratch for strata_moe_permute_static: the per-chunk histogram of
// the grouping, sized once at compile time so that callers without a device
// allocator can group slots.  One copy per device (a __device__ variable).
static __device__ __align__(256) int32_t g_permute_scratch[STRATA_PERMUTE_STATIC_SCRATCH_INTS];

// Device address of g_permute_scratch on the current device, looked up once
// per device and cached (nullptr if the lookup fails).
static int32_t* permute_scratch_ptr() {
  static std::mutex mu;
  static int32_t* cache[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int32_t*>(p);
  }
  return cache[dev];
}

strata_status_t strata_moe_permute_static(const int32_t* topk_ids, strata_moe_dims_t dims,
                                          int32_t* counts, int32_t* offsets,
                                          int32_t* sorted_token, int32_t* slot_row,
                                          strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return STRATA_ERR_INVALID_ARG;
  // The scratch limit is checked before any CUDA call, so an oversized input
  // is rejected without touching the device.
  if (permute_scratch(dims) > sizeof(int32_t) * (size_t)STRATA_PERMUTE_STATIC_SCRATCH_INTS)
    return STRATA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dims.T == 0) {
    if (cudaMemsetAsync(counts, 0, (size_t)dims.E * 4, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (size_t)(dims.E + 1) * 4, s) != cudaSuccess)
      return STRATA_ERR_CUDA;
    return STRATA_OK;
  }
  if (!ok_ptr(topk_ids) || !ok_ptr(sorted_token) || !ok_ptr(slot_row)) return STRATA_ERR_INVALID_ARG;
  int32_t* hist = permute_scratch_ptr();
  unsigned* err = check_word_ptr();
  if (!hist || !err) return STRATA_ERR_CUDA;
  return cuda_status(launch_permute(topk_ids, dims.T, dims.k, dims.E, counts, offsets,
                                    sorted_token, slot_row, hist, err, s));
}

strata_status_t strata_moe_expert_gemm_q4(strata_moe_op_t op, const uint16_t* a,
                                          const int32_t* sorted_token, const int32_t* offsets,
                                          strata_q4_t w0, strata_q4_t w1,
                                          const float* row_scale, strata_moe_dims_t dims,
                                          uint16_t* out, void* ws, size_t ws_bytes,
                                          strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (op != STRATA_OP_GATE_UP_SWIGLU && op != STRATA_OP_DOWN) return STRATA_ERR_INVALID_ARG;
  if (dims.T == 0) return STRATA_OK;
  if (!ok_ptr(a) || !ok_ptr(offsets) || !ok_ptr(w0.q) || !ok_ptr(w0.s) || !ok_ptr(out))
    return STRATA_ERR_INVALID_ARG;
  if (op == STRATA_OP_GATE_UP_SWIGLU &&
      (!ok_ptr(sorted_token) || !ok_ptr(w1.q) || !ok_ptr(w1.s) || row_scale != nullptr))
    return STRATA_ERR_INVALID_ARG;
  if (op == STRATA_OP_DOWN && !ok_opt(row_scale)) return STRATA_ERR_INVALID_ARG;
  if (!ok_ptr(ws) || ws_bytes < gemm_scratch(dims)) return STRATA_ERR_WORKSPACE;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Layout L;
  const SchedRegions r = add_schedule(L, dims);
  const Region x16 = L.add(x16_bytes(dims));
  const Schedule sch = schedule_at(static_cast<uint8_t*>(ws), r);
  if (launch_schedule(offsets, dims.E, dims.T * dims.k, kTileRows, sch, err, s) != cudaSuccess)
    return STRATA_ERR_CUDA;
  return do_gemm(op == STRATA_OP_GATE_UP_SWIGLU ? 0 : 1, a, sorted_token, offsets, w0, w1,
                 row_scale, dims, out, sch,
                 reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + x16.off), err, s);
}

strata_status_t strata_moe_combine(const uint16_t* rows, const float* topk_w,
                                   const int32_t* slot_row, strata_moe_dims_t dims, uint16_t* y,
                                   strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (dims.T == 0) return STRATA_OK;
  if (!ok_ptr(rows) || !ok_opt(topk_w) || !ok_ptr(slot_row) || !ok_ptr(y))
    return STRATA_ERR_INVALID_ARG;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  return cuda_status(launch_combine_checked(rows, topk_w, slot_row, dims.T, dims.k, dims.d, y,
                                            err, reinterpret_cast<cudaStream_t>(stream)));
}

strata_status_t strata_moe_forward(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                   strata_q4_t gate, strata_q4_t up, strata_q4_t down,
                                   strata_moe_dims_t dims, uint16_t* y, int32_t* topk_ids_out,
                                   float* topk_w_out, void* ws, size_t ws_bytes,
                                   strata_stream_t stream) {
  strata_status_t st = check_dims(dims);
  if (st != STRATA_OK) return st;
  if (dims.T == 0) return STRATA_OK;
  if (!ok_ptr(x) || !ok_ptr(w_router) || !ok_opt(bias) || !ok_ptr(gate.q) || !ok_ptr(gate.s) ||
      !ok_ptr(up.q) || !ok_ptr(up.s) || !ok_ptr(down.q) || !ok_ptr(down.s) || !ok_ptr(y) ||
      !ok_opt(topk_ids_out) || !ok_opt(topk_w_out))
    return STRATA_ERR_INVALID_ARG;
  const ForwardLayout f = forward_layout(dims);
  if (!ok_ptr(ws) || ws_bytes < f.total) return STRATA_ERR_WORKSPACE;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto at = [base](const Region& r) { return base + r.off; };
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(at(f.ids));
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(at(f.w));
  int32_t* counts = reinterpret_cast<int32_t*>(at(f.counts));
  int32_t* offsets = reinterpret_cast<int32_t*>(at(f.offsets));
  int32_t* sorted_token = reinterpret_cast<int32_t*>(at(f.sorted_token));
  int32_t* slot_row = reinterpret_cast<int32_t*>(at(f.slot_row));
  uint16_t* h = reinterpret_cast<uint16_t*>(at(f.h));
  uint16_t* rows = reinterpret_cast<uint16_t*>(at(f.rows));
  const Schedule sch = schedule_at(base, f.sched);

  if (decode_fused_fits(dims.T, dims.d, dims.E, dims.k, dims.n, dims.group)) {
    // a decode / verify batch: the whole layer in one persistent launch
    const cudaError_t e = launch_decode_fused(
        x, w_router, bias, gate.q, gate.s, up.q, up.s, down.q, down.s, dims.T, dims.d, dims.E,
        dims.k, dims.n, dims.group, y, topk_ids_out, topk_w_out, at(f.fused), err, s);
    if (e != cudaErrorNotSupported) return cuda_status(e);
  }
  st = do_route(x, w_router, bias, dims, ids, w, nullptr, reinterpret_cast<float*>(at(f.partial)),
                err, s);
  if (st != STRATA_OK) return st;
  if (launch_permute(ids, dims.T, dims.k, dims.E, counts, offsets, sorted_token, slot_row,
                     reinterpret_cast<int32_t*>(at(f.hist)), err, s) != cudaSuccess)
    return STRATA_ERR_CUDA;
  if (launch_schedule(offsets, dims.E, dims.T * dims.k, kTileRows, sch, err, s) != cudaSuccess)
    return STRATA_ERR_CUDA;
  uint16_t* x16 = reinterpret_cast<uint16_t*>(at(f.x16));
  // h is internal here: it passes between the GEMMs in the interleaved
  // feature order the down projection's dequantisation produces
  st = do_gemm(0, x, sorted_token, offsets, gate, up, nullptr, dims, h, sch, x16, err, s, true);
  if (st != STRATA_OK) return st;
  const strata_q4_t none = {nullptr, nullptr};
  st = do_gemm(1, h, nullptr, offsets, down, none, nullptr, dims, rows, sch, x16, err, s, true);
  if (st != STRATA_OK) return st;
  return cuda_status(launch_combine_checked(rows, w, slot_row, dims.T, dims.k, dims.d, y, err, s));
}

strata_status_t strata_moe_gather_rows(const uint16_t* src, const int32_t* index,
                                       int32_t src_rows, int32_t rows, int32_t width,
                                       uint16_t* dst, strata_stream_t stream) {
  if (src_rows < 0 || rows < 0 || width <= 0 || width % 8) return STRATA_ERR_INVALID_ARG;
  if (rows == 0) return STRATA_OK;
  if (src_rows == 0 || !ok_ptr(src) || !ok_ptr(index) || !ok_ptr(dst)) return STRATA_ERR_INVALID_ARG;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  return cuda_status(launch_gather_rows(src, index, src_rows, rows, width, dst, err,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

static strata_status_t check_attn_dims(const strata_attn_dims_t& a) {
  if (a.T < 0 || a.L <= 0 || a.Hq <= 0 || a.Hkv <= 0 || a.P <= 0 || a.Hq % a.Hkv)
    return STRATA_ERR_INVALID_ARG;
  if ((a.D != 64 && a.D != 128) || a.Hq / a.Hkv > 16 || a.P > 65536)
    return STRATA_ERR_UNSUPPORTED;
  return STRATA_OK;
}

size_t strata_sparse_attention_workspace_bytes(strata_attn_dims_t dims) {
  if (check_attn_dims(dims) != STRATA_OK) return 0;
  return sparse_attn_scratch(dims.T, dims.Hq, dims.P, dims.D) + 256;
}

strata_status_t strata_sparse_attention(const uint16_t* q, const uint16_t* k_cache,
                                        const uint16_t* v_cache, const int32_t* idx,
                                        strata_attn_dims_t dims, float scale, uint16_t* out,
                                        void* ws, size_t ws_bytes, strata_stream_t stream) {
  strata_status_t st = check_attn_dims(dims);
  if (st != STRATA_OK) return st;
  if (dims.T == 0) return STRATA_OK;
  if (!ok_ptr(q) || !ok_ptr(k_cache) || !ok_ptr(v_cache) || !ok_ptr(idx) || !ok_ptr(out))
    return STRATA_ERR_INVALID_ARG;
  if (!ok_ptr(ws) || ws_bytes < sparse_attn_scratch(dims.T, dims.Hq, dims.P, dims.D))
    return STRATA_ERR_WORKSPACE;
  unsigned* err = check_word_ptr();
  if (!err) return STRATA_ERR_CUDA;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)dims.D);
  return cuda_status(launch_sparse_attn(q, k_cache, v_cache, idx, dims.T, dims.L, dims.Hq,
                                        dims.Hkv, dims.D, dims.P, scale, out, ws, err,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

strata_status_t strata_moe_device_status(strata_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STRATA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_check_word, sizeof v) != cudaSuccess) return STRATA_ERR_CUDA;
  if (v == 0) return STRATA_OK;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_check_word, &zero, sizeof zero) != cudaSuccess) return STRATA_ERR_CUDA;
  return STRATA_ERR_DEVICE_CHECK;
}

}  // extern "C"
