// sq_calib.cu -- the calibration declared in include/sq_calib.h: running fp64
// sums over the traces on the device (one HBM-bound kernel per call), the
// per-head tables (phi, c, sigma2) in one kernel, the width allocation on the
// host.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <queue>
#include <vector>

#include "sq.h"
#include "sq_calib.h"
#include "sq_host.h"

using sqi::cuda_fail;
using sqi::fail;

namespace sqc {

constexpr int kSumThreads = 256;
constexpr int kSumBatch = 8;     // samples whose loads are issued before their additions
constexpr int kTabThreads = 256;

template <int VEC>
__device__ __forceinline__ void load_stream(const float* p, float (&f)[VEC]) {
  if constexpr (VEC == 4) {
    const float4 x = __ldcs(reinterpret_cast<const float4*>(p));
    f[0] = x.x;
    f[1] = x.y;
    f[2] = x.z;
    f[3] = x.w;
  } else {
    f[0] = __ldcs(p);
  }
}

template <bool SQUARE>
__device__ __forceinline__ double accumulate(double a, float x) {
  const double y = x;
  return __dadd_rn(a, SQUARE ? __dmul_rn(y, y) : y);  // y*y is exact in fp64
}

// acc[e] += f(x[t * E + e]) for t = 0 .. n-1 in order, in fp64, with f the
// square (second moments) or the identity (gate sums). A thread owns VEC
// consecutive entries and keeps their sums in registers across all samples,
// so every entry is summed in trace order whatever the grid; the trace is
// read once, streaming, kSumBatch samples in flight per thread.
template <int VEC, bool SQUARE>
__global__ void __launch_bounds__(kSumThreads) k_trace_sum(const float* __restrict__ x, int64_t n, int64_t E,
                                                          double* __restrict__ acc) {
  const int64_t e0 = ((int64_t)blockIdx.x * kSumThreads + threadIdx.x) * VEC;
  if (e0 >= E) return;
  double a[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) a[v] = acc[e0 + v];
  const float* p = x + e0;
  int64_t t = 0;
  for (; t + kSumBatch <= n; t += kSumBatch, p += kSumBatch * E) {
    float f[kSumBatch][VEC];
#pragma unroll
    for (int u = 0; u < kSumBatch; ++u) load_stream<VEC>(p + u * E, f[u]);
#pragma unroll
    for (int u = 0; u < kSumBatch; ++u)
#pragma unroll
      for (int v = 0; v < VEC; ++v) a[v] = accumulate<SQUARE>(a[v], f[u][v]);
  }
  for (; t < n; ++t, p += E) {
    float f[VEC];
    load_stream<VEC>(p, f);
#pragma unroll
    for (int v = 0; v < VEC; ++v) a[v] = accumulate<SQUARE>(a[v], f[v]);
  }
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[e0 + v] = a[v];
}

// Sum or maximum over the block; every thread gets the same value (the
// warps' partials are combined in one fixed order by every thread).
__device__ double block_reduce(double x, bool is_max, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const double y = __shfl_xor_sync(0xffffffffu, x, o);
    x = is_max ? fmax(x, y) : __dadd_rn(x, y);
  }
  __syncthreads();  // the previous reduction's readers are done with red
  if (lane == 0) red[warp] = x;
  __syncthreads();
  double r = red[0];
  for (int i = 1; i < kTabThreads / 32; ++i) r = is_max ? fmax(r, red[i]) : __dadd_rn(r, red[i]);
  return r;
}

// One value head per CTA: row impact phi from the queries' mean squares, the
// impact-weighted column scales c, and the mean square of T = S / c per unit
// (the head, or each key row). M2: [h_v][D][D] fp64 sums of S^2 over
// n_states samples; Q2: [h_k][D] fp64 sums of q^2 over n_q tokens.
template <int D>
__global__ void __launch_bounds__(kTabThreads) k_calib_tables(const double* __restrict__ M2,
                                                             const double* __restrict__ Q2, double n_states,
                                                             double n_q, int group, int per_row,
                                                             float* __restrict__ phi_out,
                                                             float* __restrict__ c_out,
                                                             double* __restrict__ sigma2_out) {
  __shared__ double red[kTabThreads / 32];
  __shared__ double w_sh[D];    // phi_i^2 of the fp32 phi
  __shared__ double ic2_sh[D];  // 1 / c_j^2 of the fp32 c
  const int h = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const double* m2 = M2 + (size_t)h * D * D;
  const double* q2 = Q2 + (size_t)(h / group) * D;

  // phi: square root of the raw impact, floored at 1e-6 of the head's largest,
  // geometric mean one
  const double s = tid < D ? q2[tid] / n_q : 0.0;
  const double top = block_reduce(s, true, red);
  float phi = 1.f;
  if (top > 0) {
    double x = 0.0, lg = 0.0;
    if (tid < D) {
      const double floor_s = 1e-6 * top;
      x = sqrt(s < floor_s ? floor_s : s);  // a NaN stays NaN
      lg = log(x);
    }
    const double gm = exp(block_reduce(lg, false, red) / D);
    phi = (float)(x / gm);
  }
  if (tid < D) {
    phi_out[(size_t)h * D + tid] = phi;
    const double p = phi;
    w_sh[tid] = __dmul_rn(p, p);
  }
  __syncthreads();

  // c: square root of the impact-weighted column RMS, floored at 1e-12 of the
  // head's largest, geometric mean one
  const double W = block_reduce(tid < D ? w_sh[tid] : 0.0, false, red);
  double rho = 0.0;
  if (tid < D) {
    double num = 0.0;
    for (int i = 0; i < D; ++i) num = __dadd_rn(num, __dmul_rn(w_sh[i], m2[(size_t)i * D + tid]));
    rho = sqrt(num / (n_states * W));
  }
  const double rtop = block_reduce(rho, true, red);
  float c = 1.f;
  if (rtop > 0) {
    double y = 0.0, lg = 0.0;
    if (tid < D) {
      const double floor_r = 1e-12 * rtop;
      y = sqrt(rho < floor_r ? floor_r : rho);
      lg = log(y);
    }
    const double gm = exp(block_reduce(lg, false, red) / D);
    c = (float)(y / gm);
  }
  if (tid < D) {
    c_out[(size_t)h * D + tid] = c;
    const double cc = c;
    ic2_sh[tid] = 1.0 / __dmul_rn(cc, cc);
  }
  __syncthreads();

  // sigma2: mean of M2_ij / c_j^2 over the unit's entries and the samples
  double head = 0.0;
  for (int i = warp; i < D; i += kTabThreads / 32) {
    double r = 0.0;
    for (int j = lane; j < D; j += 32) r = __dadd_rn(r, __dmul_rn(m2[(size_t)i * D + j], ic2_sh[j]));
#pragma unroll
    for (int o = 16; o; o >>= 1) r = __dadd_rn(r, __shfl_xor_sync(0xffffffffu, r, o));
    if (per_row && lane == 0) sigma2_out[(size_t)h * D + i] = r / (n_states * D);
    head = __dadd_rn(head, r);
  }
  if (!per_row) {
    const double total = block_reduce(lane == 0 ? head : 0.0, false, red);
    if (tid == 0) sigma2_out[h] = total / (n_states * D * D);
  }
}

}  // namespace sqc

struct sq_calib_trace {
  int h_v = 0, h_k = 0, d = 0, gate = 0, device = 0;
  size_t n_units = 0;
  int64_t n_states = 0, n_q = 0, n_g = 0;
  void* block = nullptr;
  double* m2 = nullptr;     // [h_v][d][d]
  double* q2 = nullptr;     // [h_k][d]
  double* gsum = nullptr;   // [n_units]
  float* phi = nullptr;     // [h_v][d]
  float* c = nullptr;       // [h_v][d]
  double* sigma2 = nullptr; // [n_units]
};

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

template <bool SQUARE>
sq_status launch_sum(const float* x, int64_t n, int64_t E, double* acc, cudaStream_t st) {
  const bool vec = (E % 4 == 0) && aligned16(x);
  const int64_t threads = vec ? E / 4 : E;
  const unsigned grid = (unsigned)((threads + sqc::kSumThreads - 1) / sqc::kSumThreads);
  if (vec)
    sqc::k_trace_sum<4, SQUARE><<<grid, sqc::kSumThreads, 0, st>>>(x, n, E, acc);
  else
    sqc::k_trace_sum<1, SQUARE><<<grid, sqc::kSumThreads, 0, st>>>(x, n, E, acc);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, "trace sum launch");
}

// The width allocation of include/sq_calib.h on N units. Raises all cost the
// same unit count of bits only when the allowed widths are equally spaced;
// the loop below does not rely on it: a raise that does not fit the
// remaining budget never fits later (the budget only shrinks and a unit's
// next raise only changes when it is taken), so it is dropped for good.
void allocate(const std::vector<double>& s2, const std::vector<double>& w, const std::vector<int>& widths,
              int nominal, double pivot_frac, int8_t* bits_out, uint8_t* pivot_out) {
  const size_t n = s2.size();
  const int lo = widths.front(), hi = widths.back();
  int next[9] = {0};
  for (size_t k = 0; k + 1 < widths.size(); ++k) next[widths[k]] = widths[k + 1];
  auto dist = [&](size_t u, int b) { return w[u] * s2[u] * std::ldexp(1.0, -2 * b); };

  const size_t n_piv = (size_t)std::floor(pivot_frac * (double)n + 0.5);
  std::vector<size_t> order(n);
  for (size_t u = 0; u < n; ++u) order[u] = u;
  std::sort(order.begin(), order.end(), [&](size_t a, size_t b) {
    const double da = dist(a, hi), db = dist(b, hi);
    return da > db || (da == db && a < b);
  });
  std::vector<uint8_t> piv(n, 0);
  std::vector<int> bits(n, lo);
  for (size_t k = 0; k < n_piv && k < n; ++k) {
    piv[order[k]] = 1;
    bits[order[k]] = hi;
  }
  int64_t budget = (int64_t)nominal * (int64_t)n;
  for (size_t u = 0; u < n; ++u) budget -= bits[u];

  struct Raise {
    double gain;
    size_t u;
  };
  auto lower = [](const Raise& a, const Raise& b) { return a.gain < b.gain || (a.gain == b.gain && a.u > b.u); };
  std::priority_queue<Raise, std::vector<Raise>, decltype(lower)> heap(lower);
  auto push = [&](size_t u) {
    if (piv[u] || bits[u] == hi) return;
    heap.push({dist(u, bits[u]) - dist(u, next[bits[u]]), u});
  };
  for (size_t u = 0; u < n; ++u) push(u);
  while (!heap.empty()) {
    const Raise r = heap.top();
    heap.pop();
    const int step = next[bits[r.u]] - bits[r.u];
    if (step > budget) continue;
    budget -= step;
    bits[r.u] = next[bits[r.u]];
    push(r.u);
  }
  for (size_t u = 0; u < n; ++u) {
    bits_out[u] = (int8_t)bits[u];
    pivot_out[u] = piv[u];
  }
}

// The allowed widths of a budget, ascending, after checking the budget.
sq_status check_budget(const sq_calib_budget* budget, std::vector<int>& widths) {
  widths.clear();
  for (int b = 0; b < 31; ++b) {
    if (!(budget->widths_mask >> b & 1)) continue;
    if (b != 2 && b != 4 && b != 6 && b != 8) return fail(SQ_ERR_INVALID_ARG, "width %d not in {2,4,6,8}", b);
    widths.push_back(b);
  }
  if (widths.empty()) return fail(SQ_ERR_INVALID_ARG, "widths_mask allows no width");
  if (budget->nominal_bits < widths.front() || budget->nominal_bits > widths.back())
    return fail(SQ_ERR_INVALID_ARG, "nominal_bits %d outside [%d, %d]", budget->nominal_bits, widths.front(),
                widths.back());
  if (!(budget->pivot_frac >= 0.0 && budget->pivot_frac <= 1.0))
    return fail(SQ_ERR_INVALID_ARG, "pivot_frac must be in [0, 1]");
  return SQ_OK;
}

}  // namespace

extern "C" {

sq_status sq_calib_allocate(const double* sigma2, const double* weight, int64_t n, const sq_calib_budget* budget,
                            int8_t* unit_bits, uint8_t* pivot_mask) {
  sqi::g_last_error.clear();
  if (!budget || n < 0) return fail(SQ_ERR_INVALID_ARG, "budget must not be NULL and n must be >= 0");
  if (n > 0 && (!sigma2 || !weight || !unit_bits || !pivot_mask))
    return fail(SQ_ERR_INVALID_ARG, "sigma2, weight, unit_bits and pivot_mask are required");
  std::vector<int> widths;
  const sq_status bs = check_budget(budget, widths);
  if (bs != SQ_OK) return bs;
  std::vector<double> s2(sigma2, sigma2 + n), w(weight, weight + n);
  for (int64_t u = 0; u < n; ++u)
    if (!(std::isfinite(s2[u]) && s2[u] >= 0.0 && std::isfinite(w[u]) && w[u] >= 0.0))
      return fail(SQ_ERR_INVALID_ARG, "unit %lld: sigma2 and weight must be finite and >= 0", (long long)u);
  allocate(s2, w, widths, budget->nominal_bits, budget->pivot_frac, unit_bits, pivot_mask);
  return SQ_OK;
}

sq_status sq_calib_begin(const sq_state_desc* desc, void* stream, sq_calib_trace** out) {
  sqi::g_last_error.clear();
  if (!out) return fail(SQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!desc) return fail(SQ_ERR_INVALID_ARG, "desc is NULL");
  if (desc->h_v <= 0 || desc->h_k <= 0) return fail(SQ_ERR_INVALID_ARG, "h_v and h_k must be positive");
  if (desc->h_v % desc->h_k != 0) return fail(SQ_ERR_INVALID_ARG, "h_v must be a multiple of h_k");
  if (desc->d_k != desc->d_v) return fail(SQ_ERR_UNSUPPORTED, "d_k != d_v");
  if (desc->d_k != 32 && desc->d_k != 64 && desc->d_k != 128)
    return fail(SQ_ERR_UNSUPPORTED, "d must be 32, 64 or 128 (got %d)", desc->d_k);
  if (desc->gate != SQ_GATE_HEAD && desc->gate != SQ_GATE_KEY_CHANNEL)
    return fail(SQ_ERR_INVALID_ARG, "gate must be SQ_GATE_HEAD or SQ_GATE_KEY_CHANNEL");
  auto* t = new sq_calib_trace;
  t->h_v = desc->h_v;
  t->h_k = desc->h_k;
  t->d = desc->d_k;
  t->gate = desc->gate;
  t->n_units = desc->gate == SQ_GATE_KEY_CHANNEL ? (size_t)t->h_v * t->d : (size_t)t->h_v;
  cudaError_t e = cudaGetDevice(&t->device);
  if (e != cudaSuccess) {
    delete t;
    return cuda_fail(e, "cudaGetDevice");
  }
  const size_t hvd = (size_t)t->h_v * t->d;
  const size_t sz_m2 = round256(hvd * t->d * 8), sz_q2 = round256((size_t)t->h_k * t->d * 8);
  const size_t sz_g = round256(t->n_units * 8), sz_f = round256(hvd * 4);
  const size_t total = sz_m2 + sz_q2 + 2 * sz_g + 2 * sz_f;
  e = cudaMalloc(&t->block, total);
  if (e != cudaSuccess) {
    delete t;
    (void)cudaGetLastError();
    return fail(SQ_ERR_OOM, "cudaMalloc of %zu bytes for the calibration trace failed", total);
  }
  uint8_t* b = static_cast<uint8_t*>(t->block);
  t->m2 = reinterpret_cast<double*>(b);
  b += sz_m2;
  t->q2 = reinterpret_cast<double*>(b);
  b += sz_q2;
  t->gsum = reinterpret_cast<double*>(b);
  b += sz_g;
  t->sigma2 = reinterpret_cast<double*>(b);
  b += sz_g;
  t->phi = reinterpret_cast<float*>(b);
  b += sz_f;
  t->c = reinterpret_cast<float*>(b);
  e = cudaMemsetAsync(t->block, 0, total, as_stream(stream));
  if (e != cudaSuccess) {
    cudaFree(t->block);
    delete t;
    return cuda_fail(e, "cudaMemsetAsync");
  }
  *out = t;
  return SQ_OK;
}

sq_status sq_calib_add_states(sq_calib_trace* t, const float* S, int32_t n, void* stream) {
  sqi::g_last_error.clear();
  if (!t) return fail(SQ_ERR_INVALID_ARG, "trace is NULL");
  if (n < 0) return fail(SQ_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return SQ_OK;
  if (!S || !aligned16(S)) return fail(SQ_ERR_INVALID_ARG, "S must be a 16-byte aligned device pointer");
  const sq_status s = launch_sum<true>(S, n, (int64_t)t->h_v * t->d * t->d, t->m2, as_stream(stream));
  if (s == SQ_OK) t->n_states += n;
  return s;
}

sq_status sq_calib_add_tokens(sq_calib_trace* t, const float* q, const float* g, int32_t n, void* stream) {
  sqi::g_last_error.clear();
  if (!t) return fail(SQ_ERR_INVALID_ARG, "trace is NULL");
  if (n < 0) return fail(SQ_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return SQ_OK;
  if (!q && !g) return fail(SQ_ERR_INVALID_ARG, "q and g are both NULL");
  if ((q && !aligned16(q)) || (g && !aligned16(g)))
    return fail(SQ_ERR_INVALID_ARG, "q and g must be 16-byte aligned device pointers");
  if (q) {
    const sq_status s = launch_sum<true>(q, n, (int64_t)t->h_k * t->d, t->q2, as_stream(stream));
    if (s != SQ_OK) return s;
    t->n_q += n;
  }
  if (g) {
    const sq_status s = launch_sum<false>(g, n, (int64_t)t->n_units, t->gsum, as_stream(stream));
    if (s != SQ_OK) return s;
    t->n_g += n;
  }
  return SQ_OK;
}

sq_status sq_calib_finish(sq_calib_trace* t, const sq_calib_budget* budget, const sq_calib_out* out,
                          void* stream) {
  sqi::g_last_error.clear();
  if (!t || !budget || !out) return fail(SQ_ERR_INVALID_ARG, "trace, budget and out must not be NULL");
  if (!out->unit_bits || !out->pivot_mask || !out->col_scale || !out->row_impact)
    return fail(SQ_ERR_INVALID_ARG, "unit_bits, pivot_mask, col_scale and row_impact are required");
  if (t->n_states == 0 || t->n_q == 0 || t->n_g == 0)
    return fail(SQ_ERR_INVALID_ARG, "finish needs at least one state, one query and one gate sample");
  std::vector<int> widths;
  const sq_status bs = check_budget(budget, widths);
  if (bs != SQ_OK) return bs;

  cudaStream_t st = as_stream(stream);
  const int per_row = t->gate == SQ_GATE_KEY_CHANNEL;
  const int group = t->h_v / t->h_k;
  const double ns = (double)t->n_states, nq = (double)t->n_q;
  switch (t->d) {
    case 32:
      sqc::k_calib_tables<32><<<t->h_v, sqc::kTabThreads, 0, st>>>(t->m2, t->q2, ns, nq, group, per_row, t->phi,
                                                                   t->c, t->sigma2);
      break;
    case 64:
      sqc::k_calib_tables<64><<<t->h_v, sqc::kTabThreads, 0, st>>>(t->m2, t->q2, ns, nq, group, per_row, t->phi,
                                                                   t->c, t->sigma2);
      break;
    default:
      sqc::k_calib_tables<128><<<t->h_v, sqc::kTabThreads, 0, st>>>(t->m2, t->q2, ns, nq, group, per_row,
                                                                    t->phi, t->c, t->sigma2);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "calibration tables launch");
  const size_t hvd = (size_t)t->h_v * t->d, nu = t->n_units;
  std::vector<double> s2(nu), gs(nu);
  if ((e = cudaMemcpyAsync(out->row_impact, t->phi, hvd * 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(out->col_scale, t->c, hvd * 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(s2.data(), t->sigma2, nu * 8, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(gs.data(), t->gsum, nu * 8, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess)
    return cuda_fail(e, "calibration tables copy");
  for (size_t i = 0; i < hvd; ++i) {
    if (!(std::isfinite(out->row_impact[i]) && out->row_impact[i] > 0.f) ||
        !(std::isfinite(out->col_scale[i]) && out->col_scale[i] > 0.f))
      return fail(SQ_ERR_INVALID_ARG, "the trace holds non-finite values (phi or c at %zu)", i);
  }
  std::vector<double> w(nu);
  for (size_t u = 0; u < nu; ++u) {
    if (!std::isfinite(s2[u]) || !std::isfinite(gs[u]))
      return fail(SQ_ERR_INVALID_ARG, "the trace holds non-finite values (unit %zu)", u);
    const double gm = std::min(gs[u] / (double)t->n_g, 1.0 - 1e-6);
    w[u] = 1.0 / (1.0 - gm);
  }
  allocate(s2, w, widths, budget->nominal_bits, budget->pivot_frac, out->unit_bits, out->pivot_mask);
  if (out->unit_sigma2) std::copy(s2.begin(), s2.end(), out->unit_sigma2);
  if (out->unit_weight) std::copy(w.begin(), w.end(), out->unit_weight);
  return SQ_OK;
}

sq_status sq_calib_free(sq_calib_trace* t) {
  sqi::g_last_error.clear();
  if (!t) return SQ_OK;
  cudaError_t e = cudaDeviceSynchronize();
  const cudaError_t e2 = cudaFree(t->block);
  delete t;
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  if (e2 != cudaSuccess) return cuda_fail(e2, "cudaFree");
  return SQ_OK;
}

}  // extern "C"
