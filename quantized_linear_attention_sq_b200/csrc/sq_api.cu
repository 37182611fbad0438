// sq_api.cu -- host side of the C ABI declared in include/sq.h: argument
// validation, record layout, device tables and kernel launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <mutex>
#include <vector>

#include "sq.h"
#include "sq_host.h"
#include "sq_kernels.cuh"
#include "sq_prefill.cuh"
#include "sq_step.cuh"
#include "sq_window.cuh"

namespace sqi {

thread_local std::string g_last_error;

sq_status fail(sq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

}  // namespace sqi

using sqi::cuda_fail;
using sqi::fail;
using sqi::g_last_error;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint64_t round_up(uint64_t x, uint64_t m) { return (x + m - 1) / m * m; }

// The row-impact factor as the kernels use it: a clip ratio min(phi, 1).
// A factor above 1 would set a row scale beyond what the row's largest
// entry needs; rounding that entry to a code can then give back a larger
// value, and since the next step's scale is taken from it, the row grows
// step after step. Capped at 1, the factor only ever clips rows whose
// measured impact on the readout is low.
inline float clip_ratio(float phi) { return phi < 1.0f ? phi : 1.0f; }

// Tiles per scheduling chunk of the packed step (a CTA claims this many
// consecutive head-major tiles at a time). With tiles numbered head major,
// claims of one CTA stay on one head for long runs even at one tile per
// claim, and single-tile claims balance the end of the launch best (KDA
// layer: 0.1975 ms against 0.2010 with two and 0.2040 with four; GDN
// unchanged).
constexpr int kStepChunk = 1;

// Limit of the kernels' bounded waits (a stage's data, the partials buffer).
constexpr uint64_t kWaitNs = 2000000000ull;

}  // namespace

struct sq_handle {
  sq_state_desc desc{};
  int d = 0;
  int device = 0;
  int num_sms = 0;
  // host copies of the layout
  std::vector<uint32_t> rec_off, rec_bytes;
  std::vector<uint16_t> row_off;
  std::vector<uint8_t> row_code;
  uint64_t slot_bytes = 0, pool_bytes = 0, max_rec = 0;
  // device tables (one allocation)
  void* dev_block = nullptr;
  sqk::Tables tables{};
  // launch configuration of the step kernel
  int step_grid = 0;
  int nstage = 0;
  uint32_t rec_cap = 0, stage_bytes = 0;
  uint64_t stage_rec = 0;  // largest record that goes through a stage
  size_t step_smem = 0;
  uint64_t launches = 0;
  uint64_t wait_ns = kWaitNs;     // limit of the kernels' bounded waits
  uint32_t test_extra_tx = 0;     // testing only (sq_test_stall_stage)
  // sq_decode_step_host: two device staging sets used in turn, the internal
  // stream their host-to-device copies run on, and the events that order
  // the copies after the step that last read a set.
  struct HostStage {
    void* block = nullptr;
    int32_t cap_B = 0;
    cudaEvent_t copied = nullptr;  // the set's inputs are on the device
    cudaEvent_t read = nullptr;    // the step that used the set has run
  };
  HostStage host_stage[2];
  cudaStream_t copy_stream = nullptr;
  uint64_t host_calls = 0;
  // sq_window_step: launch plan of the last window length used
  int win_W = 0, win_grid = 0;
  uint32_t win_smem = 0;
};

namespace {

// Threads per CTA of the FP32 step, quantize and dequantize (Geo) and of
// the packed step (PGeo).
int threads_of(int d) {
  switch (d) {
    case 128: return sqk::Geo<128>::NT;
    case 64: return sqk::Geo<64>::NT;
    default: return sqk::Geo<32>::NT;
  }
}
int packed_threads_of(int d) {
  switch (d) {
    case 128: return sqk::PGeo<128>::NT;
    case 64: return sqk::PGeo<64>::NT;
    default: return sqk::PGeo<32>::NT;
  }
}
uint32_t packed_aux_of(int d) {
  switch (d) {
    case 128: return sqk::PGeo<128>::AUX;
    case 64: return sqk::PGeo<64>::AUX;
    default: return sqk::PGeo<32>::AUX;
  }
}

// Every kernel that takes dynamic shared memory is allowed the device
// maximum once; occupancy then depends only on what a launch asks for, so
// handles with different record sizes never undo each other's setting.
template <typename K>
cudaError_t allow_max_smem(K kernel, int max_smem) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem - (int)fa.sharedSizeBytes);
  if (e != cudaSuccess) return e;
  // all of the unified L1 / shared storage as shared memory, so that as
  // many CTAs fit per SM as the occupancy calculation assumes
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

template <int D>
cudaError_t allow_all(int max_smem) {
  cudaError_t e = allow_max_smem(sqk::k_decode_step_packed<D>, max_smem);
  if (e == cudaSuccess) e = allow_max_smem(sqk::k_decode_step_fp32<D>, max_smem);
  if (e == cudaSuccess) e = allow_max_smem(sqk::k_quantize<D>, max_smem);
  if (e == cudaSuccess) e = allow_max_smem(sqk::k_dequantize<D>, max_smem);
  if (e == cudaSuccess) e = allow_max_smem(sqk::k_window_step<D>, max_smem);
  return e;
}

template <int D>
const void* step_kernel(bool packed) {
  return packed ? reinterpret_cast<const void*>(sqk::k_decode_step_packed<D>)
                : reinterpret_cast<const void*>(sqk::k_decode_step_fp32<D>);
}

const void* step_kernel_of(int d, bool packed) {
  switch (d) {
    case 128: return step_kernel<128>(packed);
    case 64: return step_kernel<64>(packed);
    default: return step_kernel<32>(packed);
  }
}

// Launch plan of the persistent step kernel.
struct StepPlan {
  uint32_t rec_cap = 0, stage_bytes = 0;
  int nstage = 0;
  size_t smem = 0;
  int blocks = 0;  // CTAs per SM
};

// Packed pools: a stage holds one record (every head except the all-pivot
// ones, which the kernel reads in place) plus the tile's vectors and row
// tables; the S^T k (fp64) and o partials share one buffer of 16 d fp64
// values. Two stages; as many CTAs per SM as registers and shared memory
// allow (at most 4 at d = 128). FP32 pools: 1 CTA per SM, up to 4 stages
// (the FP32 kernel's partials buffer is 32 d fp32 values).
sq_status plan_kernel(int d, bool packed, uint64_t stage_rec, int sm_smem, int optin_smem, int reserved_smem,
                      StepPlan* p) {
  const void* kern = step_kernel_of(d, packed);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
  const size_t static_smem = fa.sharedSizeBytes;
  const int nt = packed ? packed_threads_of(d) : threads_of(d);
  p->rec_cap = (uint32_t)round_up(stage_rec < 16 ? 16 : stage_rec, 128);
  // packed: the record, 2 d bytes of slack (a row read of the widest kind
  // from a clamped offset stays inside the stage), the vectors
  p->stage_bytes = packed ? (uint32_t)round_up(p->rec_cap + 2u * d + packed_aux_of(d), 128)
                          : (uint32_t)round_up(p->rec_cap + 32u * d + 32u, 128);
  const size_t red = packed ? (size_t)16 * d * 8 : (size_t)32 * d * 4;
  const size_t dyn_max = (size_t)optin_smem - static_smem;
  int by_regs = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&by_regs, kern, nt, 0);
  if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
  if (by_regs < 1) return fail(SQ_ERR_UNSUPPORTED, "step kernel does not fit on an SM");
  p->nstage = 0;
  if (packed) {
    const int ns = sqk::kPackedStages;
    const size_t smem = (size_t)ns * p->stage_bytes + red;
    if (smem > dyn_max) return fail(SQ_ERR_UNSUPPORTED, "record too large for shared memory");
    p->nstage = ns;
    p->smem = smem;
  } else {
    const long budget = (long)sm_smem - reserved_smem - (long)static_smem;
    int ns = budget > (long)red ? (int)((size_t)(budget - (long)red) / p->stage_bytes) : 0;
    if (ns > 4) ns = 4;
    if (ns < 1) return fail(SQ_ERR_UNSUPPORTED, "record too large for shared memory");
    p->nstage = ns;
    p->smem = (size_t)ns * p->stage_bytes + red;
    if (p->smem > dyn_max) return fail(SQ_ERR_UNSUPPORTED, "record too large for shared memory");
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p->blocks, kern, nt, p->smem);
  if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
  if (p->blocks < 1) return fail(SQ_ERR_UNSUPPORTED, "step kernel does not fit on an SM");
  return SQ_OK;
}

// Thread-slot order of a head's rows for the packed step: the identity for a
// head of uniform width; for a head whose rows differ, the rows grouped by
// width (stable), so the rows a warp handles together share one code path.
void build_row_perm(const uint8_t* row_code, int d, uint8_t* perm) {
  bool uniform = true;
  for (int i = 1; i < d; ++i) uniform = uniform && row_code[i] == row_code[0];
  int s = 0;
  if (uniform) {
    for (int i = 0; i < d; ++i) perm[i] = (uint8_t)i;
    return;
  }
  const uint8_t order[5] = {2, 4, 6, 8, sqk::ROW_PIVOT};
  for (uint8_t code : order)
    for (int i = 0; i < d; ++i)
      if (row_code[i] == code) perm[s++] = (uint8_t)i;
}

// Largest record that goes through a stage: that of every head except the
// all-pivot ones.
uint64_t staged_record_bytes(const uint32_t* rec_bytes, const uint8_t* head_kind, int hv) {
  uint64_t m = 0;
  for (int hh = 0; hh < hv; ++hh)
    if (head_kind[hh] != sqk::ROW_PIVOT && rec_bytes[hh] > m) m = rec_bytes[hh];
  return m;
}

// Choose stages and grid for the persistent step kernel of a handle.
sq_status plan_step(sq_handle* h) {
  const int d = h->d;
  const bool packed = h->desc.fmt == SQ_FMT_PACKED;
  int optin = 0, sm_smem = 0, reserved = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, h->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (d == 128) e = allow_all<128>(optin);
  else if (d == 64) e = allow_all<64>(optin);
  else e = allow_all<32>(optin);
  if (e != cudaSuccess) return cuda_fail(e, "kernel attributes");
  StepPlan p;
  const uint64_t stage_rec = packed ? h->stage_rec : 4ull * d * d;
  sq_status s = plan_kernel(d, packed, stage_rec, sm_smem, optin, reserved, &p);
  if (s != SQ_OK) return s;
  h->rec_cap = p.rec_cap;
  h->stage_bytes = p.stage_bytes;
  h->nstage = p.nstage;
  h->step_smem = p.smem;
  h->step_grid = p.blocks * h->num_sms;
  return SQ_OK;
}

sq_status validate_desc(const sq_state_desc* d) {
  if (!d) return fail(SQ_ERR_INVALID_ARG, "desc is NULL");
  if (d->n_slots < 1) return fail(SQ_ERR_INVALID_ARG, "n_slots must be >= 1 (got %d)", d->n_slots);
  if (d->h_v < 1 || d->h_k < 1) return fail(SQ_ERR_INVALID_ARG, "h_v and h_k must be >= 1");
  if (d->h_v % d->h_k != 0) return fail(SQ_ERR_INVALID_ARG, "h_v (%d) must be a multiple of h_k (%d)", d->h_v, d->h_k);
  if (d->d_k != d->d_v) return fail(SQ_ERR_UNSUPPORTED, "d_k != d_v is not supported");
  if (d->d_k != 32 && d->d_k != 64 && d->d_k != 128)
    return fail(SQ_ERR_UNSUPPORTED, "d must be 32, 64 or 128 (got %d)", d->d_k);
  if (d->fmt != SQ_FMT_FP32 && d->fmt != SQ_FMT_PACKED) return fail(SQ_ERR_INVALID_ARG, "bad fmt %d", d->fmt);
  if (d->gate != SQ_GATE_HEAD && d->gate != SQ_GATE_KEY_CHANNEL) return fail(SQ_ERR_INVALID_ARG, "bad gate %d", d->gate);
  return SQ_OK;
}

}  // namespace

namespace {

// Launch the decode step on device pointers (already validated).
sq_status launch_step(sq_handle* h, void* pool, const float* q, const float* k, const float* v, const float* beta,
                      const float* g, float* o, const int32_t* slot_ids, int32_t B, void* stream) {
  sqk::StepArgs a{};
  a.pool = static_cast<uint8_t*>(pool);
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.o = o;
  a.slots = slot_ids;
  a.B = B; a.h_v = h->desc.h_v; a.h_k = h->desc.h_k; a.n_slots = h->desc.n_slots; a.gate_kind = h->desc.gate;
  a.nstage = h->nstage; a.rec_cap = h->rec_cap; a.stage_bytes = h->stage_bytes;
  a.chunk = kStepChunk;
  a.slot_bytes = h->slot_bytes;
  a.wait_ns = h->wait_ns;
  a.test_extra_tx = h->test_extra_tx;
  a.t = h->tables;
  const int n_tiles = B * h->desc.h_v;
  const int grid = n_tiles < h->step_grid ? n_tiles : h->step_grid;
  const bool packed = h->desc.fmt == SQ_FMT_PACKED;
  const int nt = packed ? packed_threads_of(h->d) : threads_of(h->d);
  cudaStream_t st = as_stream(stream);
  if (packed) {
    if (h->d == 128) sqk::k_decode_step_packed<128><<<grid, nt, h->step_smem, st>>>(a);
    else if (h->d == 64) sqk::k_decode_step_packed<64><<<grid, nt, h->step_smem, st>>>(a);
    else sqk::k_decode_step_packed<32><<<grid, nt, h->step_smem, st>>>(a);
  } else {
    if (h->d == 128) sqk::k_decode_step_fp32<128><<<grid, nt, h->step_smem, st>>>(a);
    else if (h->d == 64) sqk::k_decode_step_fp32<64><<<grid, nt, h->step_smem, st>>>(a);
    else sqk::k_decode_step_fp32<32><<<grid, nt, h->step_smem, st>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching the decode step");
  h->launches++;
  return SQ_OK;
}

}  // namespace

// ------------------------------------------------------- per-window variant
namespace {

constexpr int kMaxWindow = 64;

uint64_t window_record_bytes(int d, int gate, int W) {
  const uint64_t gd = gate == SQ_GATE_KEY_CHANNEL ? (uint64_t)d : 1u;
  return 16u + 4u * (2u * (uint64_t)W * d + round_up((uint64_t)W * gd, 4));
}

template <int D>
sq_status window_plan(sq_handle* h, int W) {
  const int gd = h->desc.gate == SQ_GATE_KEY_CHANNEL ? D : 1;
  const sqk::WLay L = sqk::window_layout(D, W, gd);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, sqk::k_window_step<D>);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if ((size_t)L.total + fa.sharedSizeBytes > (size_t)optin)
    return fail(SQ_ERR_INVALID_ARG, "window of %d tokens needs %u bytes of shared memory per CTA (device limit %d)", W,
                L.total + (unsigned)fa.sharedSizeBytes, optin);
  int blocks = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, sqk::k_window_step<D>, sqk::WGeo<D>::NT, L.total);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (blocks < 1) return fail(SQ_ERR_INVALID_ARG, "window of %d tokens does not fit on an SM", W);
  h->win_W = W;
  h->win_smem = L.total;
  h->win_grid = blocks * h->num_sms;
  return SQ_OK;
}

}  // namespace

extern "C" {

const char* sq_last_error(void) { return g_last_error.c_str(); }

const char* sq_version(void) { return "sq-b200 0.1 (sm_100a)"; }

sq_status sq_state_alloc(const sq_state_desc* desc, const sq_calib* calib, void* stream, sq_handle** out,
                         size_t* pool_bytes) {
  g_last_error.clear();
  if (!out) return fail(SQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  sq_status s = validate_desc(desc);
  if (s != SQ_OK) return s;
  const int d = desc->d_k;
  const int hv = desc->h_v;
  const bool packed = desc->fmt == SQ_FMT_PACKED;
  const bool per_row = desc->gate == SQ_GATE_KEY_CHANNEL;
  const size_t n_units = per_row ? (size_t)hv * d : (size_t)hv;
  if (packed) {
    if (!calib || !calib->unit_bits || !calib->pivot_mask || !calib->col_scale || !calib->row_impact)
      return fail(SQ_ERR_INVALID_ARG, "packed format needs all four calibration arrays");
    for (size_t u = 0; u < n_units; ++u) {
      const int b = calib->unit_bits[u];
      if (!calib->pivot_mask[u] && b != 2 && b != 4 && b != 6 && b != 8)
        return fail(SQ_ERR_INVALID_ARG, "unit %zu: bit width %d not in {2,4,6,8}", u, b);
    }
    for (size_t x = 0; x < (size_t)hv * d; ++x) {
      const float c = calib->col_scale[x], p = calib->row_impact[x];
      if (!std::isfinite(c) || !(c > 0.0f)) return fail(SQ_ERR_INVALID_ARG, "col_scale[%zu] = %g is not finite > 0", x, c);
      if (!std::isfinite(p) || !(p > 0.0f)) return fail(SQ_ERR_INVALID_ARG, "row_impact[%zu] = %g is not finite > 0", x, p);
      if (!std::isfinite(1.0f / c)) return fail(SQ_ERR_INVALID_ARG, "col_scale[%zu] = %g has no finite inverse", x, c);
    }
  }
  sq_handle* h = new sq_handle();
  h->desc = *desc;
  h->d = d;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "no usable CUDA device");
  }
  // ---- layout
  h->rec_off.resize(hv);
  h->rec_bytes.resize(hv);
  h->row_off.assign((size_t)hv * d, 0);
  h->row_code.assign((size_t)hv * d, 0);
  uint64_t off = 0;
  for (int hh = 0; hh < hv; ++hh) {
    uint64_t n = 2ull * d;
    for (int i = 0; i < d; ++i) {
      const size_t u = per_row ? (size_t)hh * d + i : (size_t)hh;
      uint8_t code;
      uint64_t rb;
      if (!packed) {
        code = sqk::ROW_PIVOT;
        rb = 0;
      } else if (calib->pivot_mask[u]) {
        code = sqk::ROW_PIVOT;
        rb = 2ull * d;
      } else {
        code = (uint8_t)calib->unit_bits[u];
        rb = (uint64_t)d * code / 8;
      }
      h->row_off[(size_t)hh * d + i] = (uint16_t)n;
      h->row_code[(size_t)hh * d + i] = code;
      n += rb;
    }
    n = round_up(n, 16);
    if (!packed) n = 4ull * d * d;
    h->rec_off[hh] = (uint32_t)off;
    h->rec_bytes[hh] = (uint32_t)n;
    if (n > h->max_rec) h->max_rec = n;
    off += n;
  }
  h->slot_bytes = off;
  h->pool_bytes = off * (uint64_t)desc->n_slots;
  // ---- device tables: rec_off, rec_bytes [hv] u32; col, icol, phi [hv*d] f32;
  //      row_off [hv*d] u16; row_code [hv*d] u8; status u32
  const size_t nhd = (size_t)hv * d;
  size_t o_rec_off = 0;
  size_t o_rec_bytes = round_up(o_rec_off + 4 * hv, 16);
  size_t o_col = round_up(o_rec_bytes + 4 * hv, 16);
  size_t o_icol = round_up(o_col + 4 * nhd, 16);
  size_t o_phi = round_up(o_icol + 4 * nhd, 16);
  size_t o_row_off = round_up(o_phi + 4 * nhd, 16);
  size_t o_row_code = round_up(o_row_off + 2 * nhd, 16);
  size_t o_row_perm = round_up(o_row_code + nhd, 16);
  size_t o_head_kind = round_up(o_row_perm + nhd, 16);
  size_t o_status = round_up(o_head_kind + hv, 16);
  size_t total = round_up(o_status + 16, 256);
  std::vector<uint8_t> host(total, 0);
  memcpy(host.data() + o_rec_off, h->rec_off.data(), 4 * hv);
  memcpy(host.data() + o_rec_bytes, h->rec_bytes.data(), 4 * hv);
  float* col = reinterpret_cast<float*>(host.data() + o_col);
  float* icol = reinterpret_cast<float*>(host.data() + o_icol);
  float* phi = reinterpret_cast<float*>(host.data() + o_phi);
  for (size_t x = 0; x < nhd; ++x) {
    col[x] = packed ? calib->col_scale[x] : 1.0f;
    volatile float c = col[x];
    icol[x] = 1.0f / c;  // IEEE single-precision division
    phi[x] = packed ? clip_ratio(calib->row_impact[x]) : 1.0f;
  }
  memcpy(host.data() + o_row_off, h->row_off.data(), 2 * nhd);
  memcpy(host.data() + o_row_code, h->row_code.data(), nhd);
  for (int hh = 0; hh < hv; ++hh)
    build_row_perm(h->row_code.data() + (size_t)hh * d, d, host.data() + o_row_perm + (size_t)hh * d);
  for (int hh = 0; hh < hv; ++hh) {  // width shared by every row of the head, else 0
    uint8_t k = packed ? h->row_code[(size_t)hh * d] : 0;
    for (int i = 1; i < d && k; ++i)
      if (h->row_code[(size_t)hh * d + i] != k) k = 0;
    host[o_head_kind + hh] = k;
  }
  h->stage_rec = packed ? staged_record_bytes(h->rec_bytes.data(), host.data() + o_head_kind, hv) : 0;
  e = cudaMalloc(&h->dev_block, total);
  if (e != cudaSuccess) {
    delete h;
    return fail(SQ_ERR_OOM, "cudaMalloc of %zu table bytes failed: %s", total, cudaGetErrorString(e));
  }
  e = cudaMemcpyAsync(h->dev_block, host.data(), total, cudaMemcpyHostToDevice, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) {
    cudaFree(h->dev_block);
    delete h;
    return cuda_fail(e, "uploading tables");
  }
  uint8_t* base = static_cast<uint8_t*>(h->dev_block);
  h->tables.rec_off = reinterpret_cast<const uint32_t*>(base + o_rec_off);
  h->tables.rec_bytes = reinterpret_cast<const uint32_t*>(base + o_rec_bytes);
  h->tables.col = reinterpret_cast<const float*>(base + o_col);
  h->tables.icol = reinterpret_cast<const float*>(base + o_icol);
  h->tables.phi = reinterpret_cast<const float*>(base + o_phi);
  h->tables.row_off = reinterpret_cast<const uint16_t*>(base + o_row_off);
  h->tables.row_code = reinterpret_cast<const uint8_t*>(base + o_row_code);
  h->tables.row_perm = reinterpret_cast<const uint8_t*>(base + o_row_perm);
  h->tables.head_kind = reinterpret_cast<const uint8_t*>(base + o_head_kind);
  h->tables.status = reinterpret_cast<uint32_t*>(base + o_status);
  h->tables.xcount = reinterpret_cast<uint32_t*>(base + o_status + 4);
  h->tables.sched = reinterpret_cast<uint32_t*>(base + o_status + 8);  // zero, and reset by every step launch
  s = plan_step(h);
  if (s != SQ_OK) {
    cudaFree(h->dev_block);
    delete h;
    return s;
  }
  *out = h;
  if (pool_bytes) *pool_bytes = (size_t)h->pool_bytes;
  return SQ_OK;
}

sq_status sq_state_free(sq_handle* h) {
  g_last_error.clear();
  if (!h) return SQ_OK;
  cudaError_t e = cudaDeviceSynchronize();
  for (auto& hs : h->host_stage) {
    if (hs.block) cudaFree(hs.block);
    if (hs.copied) cudaEventDestroy(hs.copied);
    if (hs.read) cudaEventDestroy(hs.read);
  }
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  cudaError_t e2 = cudaFree(h->dev_block);
  delete h;
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  if (e2 != cudaSuccess) return cuda_fail(e2, "cudaFree");
  return SQ_OK;
}

sq_status sq_state_bytes(const sq_handle* h, sq_bytes_report* out) {
  if (!h || !out) return fail(SQ_ERR_INVALID_ARG, "NULL argument");
  const sq_state_desc& d = h->desc;
  out->pool_bytes = h->pool_bytes;
  out->slot_bytes = h->slot_bytes;
  out->state_bytes_per_step = 2 * h->slot_bytes;
  const uint64_t dd = (uint64_t)h->d;
  const uint64_t g = d.gate == SQ_GATE_HEAD ? 1 : dd;
  out->act_bytes_per_step = 4 * (2 * (uint64_t)d.h_k * dd + (uint64_t)d.h_v * dd + (uint64_t)d.h_v +
                                 (uint64_t)d.h_v * g + (uint64_t)d.h_v * dd);
  out->bits_per_value = 8.0 * (double)h->slot_bytes / ((double)d.h_v * dd * dd);
  out->max_record_bytes = h->max_rec;
  return SQ_OK;
}

sq_status sq_head_layout(const sq_handle* h, int32_t head, uint64_t* offset, uint64_t* record_bytes) {
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (head < 0 || head >= h->desc.h_v) return fail(SQ_ERR_INVALID_ARG, "head %d out of range", head);
  if (offset) *offset = h->rec_off[head];
  if (record_bytes) *record_bytes = h->rec_bytes[head];
  return SQ_OK;
}

uint64_t sq_launch_count(const sq_handle* h) { return h ? h->launches : 0; }

sq_status sq_get_exact_count(sq_handle* h, void* stream, uint32_t* count, int32_t clear) {
  g_last_error.clear();
  if (!h || !count) return fail(SQ_ERR_INVALID_ARG, "NULL argument");
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, h->tables.xcount, 4, cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(h->tables.xcount, 0, 4, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reading the exact-sum count");
  *count = v;
  return SQ_OK;
}

sq_status sq_launch_plan(const sq_handle* h, int32_t* grid, int32_t* threads, int32_t* ctas_per_sm,
                         int32_t* stages, int32_t* smem_bytes) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  const bool packed = h->desc.fmt == SQ_FMT_PACKED;
  if (grid) *grid = h->step_grid;
  if (threads) *threads = packed ? packed_threads_of(h->d) : threads_of(h->d);
  if (ctas_per_sm) *ctas_per_sm = h->num_sms ? h->step_grid / h->num_sms : 0;
  if (stages) *stages = h->nstage;
  if (smem_bytes) *smem_bytes = (int32_t)h->step_smem;
  return SQ_OK;
}

sq_status sq_set_wait_limit(sq_handle* h, uint64_t ns) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (ns < 1000) return fail(SQ_ERR_INVALID_ARG, "wait limit %llu ns is below 1000", (unsigned long long)ns);
  h->wait_ns = ns;
  return SQ_OK;
}

sq_status sq_test_stall_stages(sq_handle* h, uint32_t extra_bytes) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (extra_bytes > 65536u) return fail(SQ_ERR_INVALID_ARG, "extra_bytes %u above 65536", extra_bytes);
  h->test_extra_tx = extra_bytes;
  return SQ_OK;
}

sq_status sq_get_status(sq_handle* h, void* stream, uint32_t* bits, int32_t clear) {
  g_last_error.clear();
  if (!h || !bits) return fail(SQ_ERR_INVALID_ARG, "NULL argument");
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, h->tables.status, 4, cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(h->tables.status, 0, 4, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  *bits = v;
  return SQ_OK;
}

#define SQ_CHECK_PTR(p, name)                                                               \
  do {                                                                                      \
    if (!(p)) return fail(SQ_ERR_INVALID_ARG, "%s is NULL", name);                         \
    if (!aligned16(p)) return fail(SQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

sq_status sq_decode_step(sq_handle* h, void* pool, const float* q, const float* k, const float* v, const float* beta,
                         const float* g, float* o, const int32_t* slot_ids, int32_t B, void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (B == 0) return SQ_OK;
  if ((int64_t)B * h->desc.h_v > (int64_t)INT32_MAX / 2) return fail(SQ_ERR_INVALID_ARG, "B too large");
  SQ_CHECK_PTR(pool, "pool");
  SQ_CHECK_PTR(q, "q");
  SQ_CHECK_PTR(k, "k");
  SQ_CHECK_PTR(v, "v");
  SQ_CHECK_PTR(o, "o");
  if (!beta) return fail(SQ_ERR_INVALID_ARG, "beta is NULL");
  if (!g) return fail(SQ_ERR_INVALID_ARG, "g is NULL");
  if (h->desc.gate == SQ_GATE_KEY_CHANNEL && !aligned16(g)) return fail(SQ_ERR_INVALID_ARG, "g is not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(SQ_ERR_INVALID_ARG, "beta/g not 4-byte aligned");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  return launch_step(h, pool, q, k, v, beta, g, o, slot_ids, B, stream);
}



sq_status sq_window_buffer_bytes(const sq_handle* h, int32_t W, uint64_t* record_bytes, uint64_t* buffer_bytes) {
  g_last_error.clear();
  if (!h || !record_bytes || !buffer_bytes) return fail(SQ_ERR_INVALID_ARG, "NULL argument");
  if (W < 1 || W > kMaxWindow) return fail(SQ_ERR_INVALID_ARG, "W must be in [1, %d] (got %d)", kMaxWindow, W);
  *record_bytes = window_record_bytes(h->d, h->desc.gate, W);
  *buffer_bytes = *record_bytes * (uint64_t)h->desc.n_slots * (uint64_t)h->desc.h_v;
  return SQ_OK;
}

sq_status sq_window_step(sq_handle* h, void* pool, void* window_buf, int32_t W, const float* q, const float* k,
                         const float* v, const float* beta, const float* g, float* o, const int32_t* slot_ids,
                         int32_t B, void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (h->desc.fmt != SQ_FMT_PACKED) return fail(SQ_ERR_INVALID_ARG, "the window step needs a packed pool");
  if (W < 1 || W > kMaxWindow) return fail(SQ_ERR_INVALID_ARG, "W must be in [1, %d] (got %d)", kMaxWindow, W);
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (B == 0) return SQ_OK;
  if ((int64_t)B * h->desc.h_v > (int64_t)INT32_MAX / 2) return fail(SQ_ERR_INVALID_ARG, "B too large");
  SQ_CHECK_PTR(pool, "pool");
  SQ_CHECK_PTR(window_buf, "window_buf");
  SQ_CHECK_PTR(q, "q");
  SQ_CHECK_PTR(k, "k");
  SQ_CHECK_PTR(v, "v");
  SQ_CHECK_PTR(o, "o");
  if (!beta) return fail(SQ_ERR_INVALID_ARG, "beta is NULL");
  if (!g) return fail(SQ_ERR_INVALID_ARG, "g is NULL");
  if (h->desc.gate == SQ_GATE_KEY_CHANNEL && !aligned16(g)) return fail(SQ_ERR_INVALID_ARG, "g is not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(SQ_ERR_INVALID_ARG, "beta/g not 4-byte aligned");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  if (h->win_W != W) {
    sq_status s = h->d == 128 ? window_plan<128>(h, W) : h->d == 64 ? window_plan<64>(h, W) : window_plan<32>(h, W);
    if (s != SQ_OK) return s;
  }
  sqk::WindowArgs a{};
  a.pool = static_cast<uint8_t*>(pool);
  a.wbuf = static_cast<uint8_t*>(window_buf);
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.o = o;
  a.slots = slot_ids;
  a.B = B; a.h_v = h->desc.h_v; a.h_k = h->desc.h_k; a.n_slots = h->desc.n_slots; a.gate_kind = h->desc.gate;
  a.W = W;
  a.slot_bytes = h->slot_bytes;
  a.wait_ns = h->wait_ns;
  a.wrec_bytes = (uint32_t)window_record_bytes(h->d, h->desc.gate, W);
  a.t = h->tables;
  const int n_tiles = B * h->desc.h_v;
  const int grid = n_tiles < h->win_grid ? n_tiles : h->win_grid;
  cudaStream_t st = as_stream(stream);
  if (h->d == 128) sqk::k_window_step<128><<<grid, sqk::WGeo<128>::NT, h->win_smem, st>>>(a);
  else if (h->d == 64) sqk::k_window_step<64><<<grid, sqk::WGeo<64>::NT, h->win_smem, st>>>(a);
  else sqk::k_window_step<32><<<grid, sqk::WGeo<32>::NT, h->win_smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching the window step");
  h->launches++;
  return SQ_OK;
}

sq_status sq_decode_step_host(sq_handle* h, void* pool, const float* q, const float* k, const float* v,
                              const float* beta, const float* g, float* o, const int32_t* slot_ids, int32_t B,
                              void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (B == 0) return SQ_OK;
  if ((int64_t)B * h->desc.h_v > (int64_t)INT32_MAX / 2) return fail(SQ_ERR_INVALID_ARG, "B too large");
  SQ_CHECK_PTR(pool, "pool");
  if (!q || !k || !v || !beta || !g || !o) return fail(SQ_ERR_INVALID_ARG, "q, k, v, beta, g and o are required");
  const size_t d = (size_t)h->d, hv = (size_t)h->desc.h_v, hk = (size_t)h->desc.h_k, nB = (size_t)B;
  const size_t b_qk = 4 * nB * hk * d, b_v = 4 * nB * hv * d, b_beta = 4 * nB * hv;
  const size_t b_g = h->desc.gate == SQ_GATE_KEY_CHANNEL ? b_v : b_beta, b_slot = 4 * nB;
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  if (!h->copy_stream) {
    if ((e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags");
    for (auto& hs : h->host_stage)
      if ((e = cudaEventCreateWithFlags(&hs.copied, cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&hs.read, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e, "cudaEventCreateWithFlags");
  }
  sq_handle::HostStage& hs = h->host_stage[h->host_calls & 1];
  // staging layout: q | k | v | o | beta | g | slot ids, 256-byte aligned pieces
  const size_t o_q = 0, o_k = round_up(b_qk, 256), o_v = o_k + round_up(b_qk, 256);
  const size_t o_o = o_v + round_up(b_v, 256), o_b = o_o + round_up(b_v, 256);
  const size_t o_g = o_b + round_up(b_beta, 256), o_s = o_g + round_up(b_g, 256);
  const size_t total = o_s + round_up(b_slot, 256);
  if (hs.cap_B < B) {
    // a larger batch than before: wait for every use of the old set, then replace it
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    if (hs.block) cudaFree(hs.block);
    hs.block = nullptr;
    hs.cap_B = 0;
    if ((e = cudaMalloc(&hs.block, total)) != cudaSuccess) {
      (void)cudaGetLastError();
      return fail(SQ_ERR_OOM, "cudaMalloc of %zu bytes of staging failed", total);
    }
    hs.cap_B = B;
  }
  uint8_t* base = static_cast<uint8_t*>(hs.block);
  float* dq = reinterpret_cast<float*>(base + o_q);
  float* dk = reinterpret_cast<float*>(base + o_k);
  float* dv = reinterpret_cast<float*>(base + o_v);
  float* dout = reinterpret_cast<float*>(base + o_o);
  float* dbeta = reinterpret_cast<float*>(base + o_b);
  float* dg = reinterpret_cast<float*>(base + o_g);
  int32_t* dslot = slot_ids ? reinterpret_cast<int32_t*>(base + o_s) : nullptr;
  // the copies of this step wait only for the step that last read this set,
  // so they overlap the step launched by the previous call
  cudaStream_t cs = h->copy_stream;
  if ((e = cudaStreamWaitEvent(cs, hs.read, 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(dq, q, b_qk, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaMemcpyAsync(dk, k, b_qk, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaMemcpyAsync(dv, v, b_v, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaMemcpyAsync(dbeta, beta, b_beta, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaMemcpyAsync(dg, g, b_g, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (slot_ids && (e = cudaMemcpyAsync(dslot, slot_ids, b_slot, cudaMemcpyHostToDevice, cs)) != cudaSuccess) ||
      (e = cudaEventRecord(hs.copied, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(st, hs.copied, 0)) != cudaSuccess)
    return cuda_fail(e, "staging the step's inputs");
  // o: written by the kernel straight into mapped page-locked host memory,
  // else staged and copied back on the caller's stream
  void* mapped = nullptr;
  const bool zero_copy = cudaHostGetDevicePointer(&mapped, o, 0) == cudaSuccess && mapped;
  if (!zero_copy) (void)cudaGetLastError();
  float* o_dev = zero_copy ? static_cast<float*>(mapped) : dout;
  sq_status s = launch_step(h, pool, dq, dk, dv, dbeta, dg, o_dev, dslot, B, stream);
  if (s != SQ_OK) return s;
  if ((e = cudaEventRecord(hs.read, st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if (!zero_copy && (e = cudaMemcpyAsync(o, dout, b_v, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e, "copying o to the host");
  h->host_calls++;
  return SQ_OK;
}

sq_status sq_quantize_state(sq_handle* h, void* pool, const float* S, const int32_t* slot_ids, int32_t B,
                            void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (B == 0) return SQ_OK;
  SQ_CHECK_PTR(pool, "pool");
  SQ_CHECK_PTR(S, "S");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  cudaStream_t st = as_stream(stream);
  const int n_tiles = B * h->desc.h_v;
  const int nt = threads_of(h->d);
  if (h->desc.fmt == SQ_FMT_FP32) {
    if (h->d == 128) sqk::k_copy_fp32<128><<<n_tiles, 256, 0, st>>>(static_cast<float*>(pool), S, nullptr, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
    else if (h->d == 64) sqk::k_copy_fp32<64><<<n_tiles, 256, 0, st>>>(static_cast<float*>(pool), S, nullptr, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
    else sqk::k_copy_fp32<32><<<n_tiles, 256, 0, st>>>(static_cast<float*>(pool), S, nullptr, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
  } else {
    sqk::QuantArgs a{};
    a.pool = static_cast<uint8_t*>(pool);
    a.S = S;
    a.slots = slot_ids;
    a.B = B; a.h_v = h->desc.h_v; a.n_slots = h->desc.n_slots;
    a.slot_bytes = h->slot_bytes;
    a.t = h->tables;
    const size_t smem = round_up(h->max_rec, 16) + 7 * (size_t)h->d;
    if (h->d == 128) sqk::k_quantize<128><<<n_tiles, nt, smem, st>>>(a);
    else if (h->d == 64) sqk::k_quantize<64><<<n_tiles, nt, smem, st>>>(a);
    else sqk::k_quantize<32><<<n_tiles, nt, smem, st>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching quantize");
  h->launches++;
  return SQ_OK;
}

sq_status sq_dequantize_state(sq_handle* h, const void* pool, float* S_out, const int32_t* slot_ids, int32_t B,
                              void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (B == 0) return SQ_OK;
  SQ_CHECK_PTR(pool, "pool");
  SQ_CHECK_PTR(S_out, "S_out");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  cudaStream_t st = as_stream(stream);
  const int n_tiles = B * h->desc.h_v;
  const int nt = threads_of(h->d);
  if (h->desc.fmt == SQ_FMT_FP32) {
    float* P = const_cast<float*>(static_cast<const float*>(pool));
    if (h->d == 128) sqk::k_copy_fp32<128><<<n_tiles, 256, 0, st>>>(P, nullptr, S_out, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
    else if (h->d == 64) sqk::k_copy_fp32<64><<<n_tiles, 256, 0, st>>>(P, nullptr, S_out, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
    else sqk::k_copy_fp32<32><<<n_tiles, 256, 0, st>>>(P, nullptr, S_out, slot_ids, h->desc.h_v, h->desc.n_slots, h->tables.status);
  } else {
    sqk::QuantArgs a{};
    a.pool = static_cast<uint8_t*>(const_cast<void*>(pool));
    a.S_out = S_out;
    a.slots = slot_ids;
    a.B = B; a.h_v = h->desc.h_v; a.n_slots = h->desc.n_slots;
    a.slot_bytes = h->slot_bytes;
    a.t = h->tables;
    const size_t smem = round_up(h->max_rec, 16);
    if (h->d == 128) sqk::k_dequantize<128><<<n_tiles, nt, smem, st>>>(a);
    else if (h->d == 64) sqk::k_dequantize<64><<<n_tiles, nt, smem, st>>>(a);
    else sqk::k_dequantize<32><<<n_tiles, nt, smem, st>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching dequantize");
  h->launches++;
  return SQ_OK;
}

sq_status sq_prefill(sq_handle* h, void* pool, const float* S0, const float* q, const float* k, const float* v,
                     const float* beta, const float* g, float* o, float* S_out, const int32_t* lengths,
                     const int32_t* slot_ids, int32_t B, int32_t L, void* stream) {
  g_last_error.clear();
  if (!h) return fail(SQ_ERR_INVALID_ARG, "NULL handle");
  if (B < 0 || L < 0) return fail(SQ_ERR_INVALID_ARG, "B and L must be >= 0 (got %d, %d)", B, L);
  if (B == 0) return SQ_OK;
  if ((int64_t)B * h->desc.h_v > (int64_t)INT32_MAX / 2) return fail(SQ_ERR_INVALID_ARG, "B too large");
  SQ_CHECK_PTR(pool, "pool");
  if (L > 0) {
    SQ_CHECK_PTR(q, "q");
    SQ_CHECK_PTR(k, "k");
    SQ_CHECK_PTR(v, "v");
    SQ_CHECK_PTR(o, "o");
    if (!beta) return fail(SQ_ERR_INVALID_ARG, "beta is NULL");
    if (!g) return fail(SQ_ERR_INVALID_ARG, "g is NULL");
    if (h->desc.gate == SQ_GATE_KEY_CHANNEL && !aligned16(g))
      return fail(SQ_ERR_INVALID_ARG, "g is not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(g) & 3u))
      return fail(SQ_ERR_INVALID_ARG, "beta/g not 4-byte aligned");
  }
  if (S0 && !aligned16(S0)) return fail(SQ_ERR_INVALID_ARG, "S0 is not 16-byte aligned");
  if (S_out && !aligned16(S_out)) return fail(SQ_ERR_INVALID_ARG, "S_out is not 16-byte aligned");
  if (lengths && (reinterpret_cast<uintptr_t>(lengths) & 3u)) return fail(SQ_ERR_INVALID_ARG, "lengths misaligned");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  sqk::PrefillArgs a{};
  a.pool = static_cast<uint8_t*>(pool);
  a.S0 = S0;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.o = o;
  a.S_out = S_out;
  a.lengths = lengths;
  a.slots = slot_ids;
  a.B = B; a.L = L; a.h_v = h->desc.h_v; a.h_k = h->desc.h_k; a.n_slots = h->desc.n_slots;
  a.gate_kind = h->desc.gate;
  a.fmt_fp32 = h->desc.fmt == SQ_FMT_FP32;
  a.slot_bytes = h->slot_bytes;
  a.t = h->tables;
  const int n_tiles = B * h->desc.h_v;
  const uint32_t rec = a.fmt_fp32 ? 0u : (uint32_t)h->max_rec;
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaSuccess;
  if (h->d == 128) {
    const size_t smem = sqk::PrefillSmem<128>::bytes(rec);
    e = cudaFuncSetAttribute(sqk::k_prefill<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) sqk::k_prefill<128><<<n_tiles, 256, smem, st>>>(a);
  } else if (h->d == 64) {
    const size_t smem = sqk::PrefillSmem<64>::bytes(rec);
    e = cudaFuncSetAttribute(sqk::k_prefill<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) sqk::k_prefill<64><<<n_tiles, 128, smem, st>>>(a);
  } else {
    const size_t smem = sqk::PrefillSmem<32>::bytes(rec);
    e = cudaFuncSetAttribute(sqk::k_prefill<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) sqk::k_prefill<32><<<n_tiles, 64, smem, st>>>(a);
  }
  if (e != cudaSuccess) return cuda_fail(e, "setting the prefill's shared memory");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching the prefill");
  h->launches++;
  return SQ_OK;
}

}  // extern "C"

// ===================================================================
// Decode step that allocates nothing (sq_decode_step_noalloc).
//
// The regular path keeps its per-head tables (record offsets, row offsets,
// widths, c, 1/c, phi, the status word) in device memory that
// sq_state_alloc obtains with cudaMalloc. Here the same tables live in one
// file-scope __device__ array, rebuilt on every call; nothing is allocated
// on the device or the host heap.
// ===================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = 160 * 1024;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Host staging for the tables (the copy from pageable memory returns only
// after the data has left this buffer, so it can be reused by the next call).
static uint8_t g_noalloc_host[kNoAllocScratchBytes];
static std::mutex g_noalloc_mutex;

constexpr int kMaxDevices = 64;
struct NoAllocDevice {
  bool ready = false;
  uint8_t* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int num_sms = 0, sm_smem = 0, optin_smem = 0, reserved_smem = 0;
};
static NoAllocDevice g_noalloc_dev[kMaxDevices];

// Once per device, with that device current: the device address of the
// scratch array (host code must not use the symbol itself) and the launch
// limits. Runs inside the first call on the device.
sq_status noalloc_setup(int dev, NoAllocDevice** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(SQ_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
  NoAllocDevice& nd = g_noalloc_dev[dev];
  if (!nd.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    nd.scratch = static_cast<uint8_t*>(p);
    e = cudaDeviceGetAttribute(&nd.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nd.sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nd.optin_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nd.reserved_smem, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e == cudaSuccess) e = allow_all<128>(nd.optin_smem);
    if (e == cudaSuccess) e = allow_all<64>(nd.optin_smem);
    if (e == cudaSuccess) e = allow_all<32>(nd.optin_smem);
    if (e != cudaSuccess) return cuda_fail(e, "no-alloc set-up");
    nd.ready = true;
  }
  *out = &nd;
  return SQ_OK;
}

}  // namespace

extern "C" sq_status sq_decode_step_noalloc(const sq_state_desc* desc, const sq_calib* calib, void* pool,
                                             const float* q, const float* k, const float* v, const float* beta,
                                             const float* g, float* o, const int32_t* slot_ids, int32_t B,
                                             uint32_t* status, void* stream) {
  g_last_error.clear();
  sq_status s = validate_desc(desc);
  if (s != SQ_OK) return s;
  if (desc->fmt != SQ_FMT_PACKED) return fail(SQ_ERR_UNSUPPORTED, "the no-alloc step takes packed pools only");
  const int d = desc->d_k, hv = desc->h_v;
  if (hv > SQ_NOALLOC_MAX_HEADS)
    return fail(SQ_ERR_UNSUPPORTED, "no-alloc step: h_v = %d exceeds its maximum of %d heads", hv,
                SQ_NOALLOC_MAX_HEADS);
  if (B < 0) return fail(SQ_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  const bool per_row = desc->gate == SQ_GATE_KEY_CHANNEL;
  const size_t n_units = per_row ? (size_t)hv * d : (size_t)hv;
  if (!calib || !calib->unit_bits || !calib->pivot_mask || !calib->col_scale || !calib->row_impact)
    return fail(SQ_ERR_INVALID_ARG, "packed format needs all four calibration arrays");
  for (size_t u = 0; u < n_units; ++u) {
    const int b = calib->unit_bits[u];
    if (!calib->pivot_mask[u] && b != 2 && b != 4 && b != 6 && b != 8)
      return fail(SQ_ERR_INVALID_ARG, "unit %zu: bit width %d not in {2,4,6,8}", u, b);
  }
  const size_t nhd = (size_t)hv * d;
  for (size_t x = 0; x < nhd; ++x) {
    const float c = calib->col_scale[x], p = calib->row_impact[x];
    if (!std::isfinite(c) || !(c > 0.0f) || !std::isfinite(1.0f / c))
      return fail(SQ_ERR_INVALID_ARG, "col_scale[%zu] = %g is not finite > 0", x, c);
    if (!std::isfinite(p) || !(p > 0.0f)) return fail(SQ_ERR_INVALID_ARG, "row_impact[%zu] = %g is not finite > 0", x, p);
  }
  if (B == 0) return SQ_OK;
  if ((int64_t)B * hv > (int64_t)INT32_MAX / 2) return fail(SQ_ERR_INVALID_ARG, "B too large");
  SQ_CHECK_PTR(pool, "pool");
  SQ_CHECK_PTR(q, "q");
  SQ_CHECK_PTR(k, "k");
  SQ_CHECK_PTR(v, "v");
  SQ_CHECK_PTR(o, "o");
  if (!beta || !g) return fail(SQ_ERR_INVALID_ARG, "beta/g is NULL");
  if (per_row && !aligned16(g)) return fail(SQ_ERR_INVALID_ARG, "g is not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(SQ_ERR_INVALID_ARG, "beta/g not 4-byte aligned");
  if (slot_ids && (reinterpret_cast<uintptr_t>(slot_ids) & 3u)) return fail(SQ_ERR_INVALID_ARG, "slot_ids misaligned");
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return fail(SQ_ERR_INVALID_ARG, "status misaligned");

  // table layout inside the scratch array (same tables as a handle's)
  const size_t o_rec_off = 0;
  const size_t o_rec_bytes = round_up(o_rec_off + 4 * (size_t)hv, 16);
  const size_t o_col = round_up(o_rec_bytes + 4 * (size_t)hv, 16);
  const size_t o_icol = round_up(o_col + 4 * nhd, 16);
  const size_t o_phi = round_up(o_icol + 4 * nhd, 16);
  const size_t o_row_off = round_up(o_phi + 4 * nhd, 16);
  const size_t o_row_code = round_up(o_row_off + 2 * nhd, 16);
  const size_t o_row_perm = round_up(o_row_code + nhd, 16);
  const size_t o_head_kind = round_up(o_row_perm + nhd, 16);
  const size_t o_status = round_up(o_head_kind + (size_t)hv, 16);
  const size_t total = round_up(o_status + 16, 16);
  if (total > kNoAllocScratchBytes)
    return fail(SQ_ERR_UNSUPPORTED, "no-alloc step: tables need %zu bytes, above its %zu-byte scratch", total,
                kNoAllocScratchBytes);

  // The tables travel by cudaMemcpyAsync from a host buffer that the next
  // call overwrites. Captured into a CUDA graph, that copy would replay
  // whatever tables the last call left there, so calls during a stream
  // capture are refused.
  {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t ce = cudaStreamIsCapturing(as_stream(stream), &cap);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone)
      return fail(SQ_ERR_UNSUPPORTED, "the no-alloc step cannot run while its stream is being captured");
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "no usable CUDA device");
  NoAllocDevice* nd = nullptr;
  s = noalloc_setup(dev, &nd);
  if (s != SQ_OK) return s;

  uint8_t* host = g_noalloc_host;
  memset(host, 0, total);
  uint32_t* rec_off = reinterpret_cast<uint32_t*>(host + o_rec_off);
  uint32_t* rec_bytes = reinterpret_cast<uint32_t*>(host + o_rec_bytes);
  float* col = reinterpret_cast<float*>(host + o_col);
  float* icol = reinterpret_cast<float*>(host + o_icol);
  float* phi = reinterpret_cast<float*>(host + o_phi);
  uint16_t* row_off = reinterpret_cast<uint16_t*>(host + o_row_off);
  uint8_t* row_code = host + o_row_code;
  uint8_t* head_kind = host + o_head_kind;
  uint64_t off = 0, max_rec = 0;
  for (int hh = 0; hh < hv; ++hh) {
    uint64_t n = 2ull * d;
    for (int i = 0; i < d; ++i) {
      const size_t u = per_row ? (size_t)hh * d + i : (size_t)hh;
      const bool piv = calib->pivot_mask[u] != 0;
      const uint8_t code = piv ? sqk::ROW_PIVOT : (uint8_t)calib->unit_bits[u];
      row_off[(size_t)hh * d + i] = (uint16_t)n;
      row_code[(size_t)hh * d + i] = code;
      n += piv ? 2ull * d : (uint64_t)d * code / 8;
    }
    n = round_up(n, 16);
    rec_off[hh] = (uint32_t)off;
    rec_bytes[hh] = (uint32_t)n;
    if (n > max_rec) max_rec = n;
    off += n;
    uint8_t kind = row_code[(size_t)hh * d];
    for (int i = 1; i < d && kind; ++i)
      if (row_code[(size_t)hh * d + i] != kind) kind = 0;
    head_kind[hh] = kind;
    build_row_perm(row_code + (size_t)hh * d, d, host + o_row_perm + (size_t)hh * d);
  }
  for (size_t x = 0; x < nhd; ++x) {
    col[x] = calib->col_scale[x];
    volatile float c = col[x];
    icol[x] = 1.0f / c;  // IEEE single-precision division
    phi[x] = clip_ratio(calib->row_impact[x]);
  }
  cudaStream_t st = as_stream(stream);
  e = cudaMemcpyAsync(nd->scratch, host, total, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "uploading no-alloc tables");

  sqk::StepArgs a{};
  a.pool = static_cast<uint8_t*>(pool);
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.o = o;
  a.slots = slot_ids;
  a.B = B; a.h_v = hv; a.h_k = desc->h_k; a.n_slots = desc->n_slots; a.gate_kind = desc->gate;
  a.slot_bytes = off;
  a.wait_ns = kWaitNs;
  a.test_extra_tx = 0;
  a.t.rec_off = reinterpret_cast<const uint32_t*>(nd->scratch + o_rec_off);
  a.t.rec_bytes = reinterpret_cast<const uint32_t*>(nd->scratch + o_rec_bytes);
  a.t.col = reinterpret_cast<const float*>(nd->scratch + o_col);
  a.t.icol = reinterpret_cast<const float*>(nd->scratch + o_icol);
  a.t.phi = reinterpret_cast<const float*>(nd->scratch + o_phi);
  a.t.row_off = reinterpret_cast<const uint16_t*>(nd->scratch + o_row_off);
  a.t.row_code = reinterpret_cast<const uint8_t*>(nd->scratch + o_row_code);
  a.t.row_perm = reinterpret_cast<const uint8_t*>(nd->scratch + o_row_perm);
  a.t.head_kind = reinterpret_cast<const uint8_t*>(nd->scratch + o_head_kind);
  a.t.status = status ? status : reinterpret_cast<uint32_t*>(nd->scratch + o_status);
  a.t.xcount = reinterpret_cast<uint32_t*>(nd->scratch + o_status + 4);
  a.t.sched = reinterpret_cast<uint32_t*>(nd->scratch + o_status + 8);  // uploaded as zeros above

  // launch plan (same rule as a handle's)
  StepPlan p;
  s = plan_kernel(d, true, staged_record_bytes(rec_bytes, head_kind, hv), nd->sm_smem, nd->optin_smem,
                  nd->reserved_smem, &p);
  if (s != SQ_OK) return s;
  a.rec_cap = p.rec_cap;
  a.stage_bytes = p.stage_bytes;
  a.nstage = p.nstage;
  a.chunk = kStepChunk;
  const size_t smem = p.smem;
  const int blocks = p.blocks;
  const int n_tiles = B * hv;
  const int grid = n_tiles < blocks * nd->num_sms ? n_tiles : blocks * nd->num_sms;
  if (!status) {
    e = cudaMemsetAsync(nd->scratch + o_status, 0, 4, st);  // the scratch status word starts at zero
    if (e != cudaSuccess) return cuda_fail(e, "clearing the scratch status word");
  }
  if (d == 128) sqk::k_decode_step_packed<128><<<grid, packed_threads_of(128), smem, st>>>(a);
  else if (d == 64) sqk::k_decode_step_packed<64><<<grid, packed_threads_of(64), smem, st>>>(a);
  else sqk::k_decode_step_packed<32><<<grid, packed_threads_of(32), smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launching the no-alloc decode step");
  return SQ_OK;
}
