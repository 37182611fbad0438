// sq_prefill.cuh -- prefill handoff: the gated delta rule run over a whole
// prompt with the state held on chip, then quantized once into the pool.
//
// One CTA per (request, value head) tile, one thread per value column: the
// column of the fp32 state lives in that thread's registers for every token
// of the prompt; each token applies exactly the arithmetic of the FP32 decode
// step (gate, S^T k column sum, delta update, S^T q column sum, with the
// step's summation order), so a prefill of L tokens equals L FP32 decode
// steps bit for bit. The vectors of the next chunk of tokens are fetched
// with cp.async into a second buffer while the current chunk runs. After
// the last token the tile is written once: quantized into the packed pool
// slot (the dual-axis quantization of the step kernels: T = S / c, row
// scales from the row maxima and phi, codes rounded to nearest even), or as
// fp32 into an FP32 pool, and optionally also as fp32 S to S_out.
// ("STEPQuant review (e-cogni)", section "Contexto": the state a prompt
// leaves behind is what every later decode step updates; the pages'
// serving flow quantizes it when it enters the state cache.)
#pragma once

#include "sq_kernels.cuh"

namespace sqk {

struct PrefillArgs {
  uint8_t* pool;          // packed pool, or fp32 S pool (fmt_fp32)
  const float* S0;        // [B, h_v, d, d] initial state, or null for zeros
  const float* q;         // [B, L, h_k, d]
  const float* k;         // [B, L, h_k, d]
  const float* v;         // [B, L, h_v, d]
  const float* beta;      // [B, L, h_v]
  const float* g;         // [B, L, h_v] or [B, L, h_v, d]
  float* o;               // [B, L, h_v, d]; rows t >= length are not written
  float* S_out;           // [B, h_v, d, d] final fp32 state, or null
  const int32_t* lengths; // [B] tokens of each prompt (clamped to [0, L]), or null for L
  const int32_t* slots;   // [B] or null
  int32_t B, L, h_v, h_k, n_slots, gate_kind, fmt_fp32;
  uint64_t slot_bytes;
  Tables t;
};

// Shared memory of one prefill CTA. During the prompt: two chunks of TC
// tokens' vectors. After it: the fp32 state (row-major, to change from the
// column-per-thread layout to the step kernels' thread map), then the record
// and the head's row tables behind it.
template <int D>
struct PrefillSmem {
  static constexpr int TC = 16;                  // tokens per staged chunk
  static constexpr int TOK = 4 * D + 8;          // floats per token: k q v g | beta g0 pad
  static constexpr int CHUNK = TC * TOK;         // floats per chunk buffer
  static constexpr size_t S_BYTES = (size_t)D * D * 4;
  static constexpr size_t TOK_BYTES = (size_t)2 * CHUNK * 4;
  // the token buffers, then the state, share [0, REGION); the record follows
  static constexpr size_t REGION = ((S_BYTES > TOK_BYTES ? S_BYTES : TOK_BYTES) + 127) / 128 * 128;
  static size_t bytes(uint32_t rec_cap) { return REGION + (rec_cap + 15) / 16 * 16 + 7 * D; }
};

// A 16-byte shared-memory load that is neither merged with an earlier load
// of the same address nor moved ahead of the other such loads: the token's
// k is read once for S^T k and once for the update, and keeping reads alive
// in registers next to the state would overflow the 128 registers a thread
// has at two CTAs per SM.
__device__ __forceinline__ float4 lds128(const float* p) {
  float4 v;
  asm volatile("ld.volatile.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Fetch tokens t0 .. t0+n-1 of tile (b, h) into `buf` (token u at
// buf + u * TOK): 16-byte pieces of k, q, v (and g per key channel), then
// beta and the per-head gate, spread over the CTA's threads.
template <int D>
__device__ __forceinline__ void prefill_fetch(const PrefillArgs& a, int b, int h, int hk, int t0, int n, float* buf) {
  using M = PrefillSmem<D>;
  constexpr int C = D / 4;
  constexpr int P = 4 * C + 2;  // pieces per token
  const bool kda = a.gate_kind != 0;
  for (int id = threadIdx.x; id < n * P; id += Geo<D>::NT) {
    const int u = id / P;
    const int w = id - u * P;
    const size_t bt = (size_t)b * a.L + t0 + u;
    float* tb = buf + u * M::TOK;
    if (w < C) {
      cp_async16(tb + 4 * w, a.k + (bt * a.h_k + hk) * D + 4 * w);
    } else if (w < 2 * C) {
      cp_async16(tb + D + 4 * (w - C), a.q + (bt * a.h_k + hk) * D + 4 * (w - C));
    } else if (w < 3 * C) {
      cp_async16(tb + 2 * D + 4 * (w - 2 * C), a.v + (bt * a.h_v + h) * D + 4 * (w - 2 * C));
    } else if (w < 4 * C) {
      if (kda) cp_async16(tb + 3 * D + 4 * (w - 3 * C), a.g + (bt * a.h_v + h) * D + 4 * (w - 3 * C));
    } else if (w == 4 * C) {
      cp_async4(tb + 4 * D, a.beta + bt * a.h_v + h);
    } else if (!kda) {
      cp_async4(tb + 4 * D + 1, a.g + bt * a.h_v + h);
    }
  }
  cp_async_commit();
}

// The column sum of the step kernels for one column held by two threads,
// this thread holding half hh of the row groups: S2[r][x] = (S[r NG + hh NG/2
// + 2x], S[r NG + hh NG/2 + 2x + 1]) of the column, vec the D per-row factors
// in shared memory. The partial of row group g is sum_r S[r NG + g]
// vec[r NG + g] (r = 0 first); a half's row groups are summed into four
// accumulators a[g & 3] in order and give (a0 + a1) + (a2 + a3); the total
// is half 0 + half 1 (the partner thread is the neighbouring lane): the same
// operations, in the same order, as the deposit and column total of the FP32
// step.
template <int D>
__device__ __forceinline__ float column_tree(const float2 (&S2)[Geo<D>::RPT][Geo<D>::NG / 4], const float* vec,
                                             int hh) {
  using G = Geo<D>;
  constexpr int PH = G::NG / 4;  // pairs of row groups per half
  // r outer, pairs inner: consecutive loads feed PH independent chains
  float2 p[PH];
#pragma unroll
  for (int r = 0; r < G::RPT; ++r)
#pragma unroll
    for (int x = 0; x < PH; x += 2) {
      const float4 kv = lds128(vec + r * G::NG + hh * (G::NG / 2) + 2 * x);
      const float2 k0 = make_float2(kv.x, kv.y), k1 = make_float2(kv.z, kv.w);
      p[x] = r == 0 ? __fmul2_rn(S2[r][x], k0) : __ffma2_rn(S2[r][x], k0, p[x]);
      p[x + 1] = r == 0 ? __fmul2_rn(S2[r][x + 1], k1) : __ffma2_rn(S2[r][x + 1], k1, p[x + 1]);
    }
  float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int x = 0; x < PH; x += 2) {
    a01 = __fadd2_rn(a01, p[x]);
    a23 = __fadd2_rn(a23, p[x + 1]);
  }
  const float t = __fadd_rn(__fadd_rn(a01.x, a01.y), __fadd_rn(a23.x, a23.y));
  return __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 1));  // t0 + t1 on both threads (addition commutes)
}

// One CTA per (request, value head) state, two threads per value column j
// (thread 2j + hh holds the column's rows of row groups hh NG/2 .. hh NG/2 +
// NG/2 - 1): the state stays in registers for the whole prompt and a token's
// two column sums need one shuffle each and no barrier (one barrier per
// chunk of TC tokens hands over the next chunk's vectors).
template <int D>
__global__ void __launch_bounds__(Geo<D>::NT, 2) k_prefill(const PrefillArgs a) {
  using G = Geo<D>;
  using M = PrefillSmem<D>;
  constexpr int NQ = G::NG / 4;  // float2 pairs per row slot and thread
  extern __shared__ __align__(128) uint8_t smem[];
  float* tok = reinterpret_cast<float*>(smem);

  const int tile = blockIdx.x;
  const int b = tile / a.h_v;
  const int h = tile - b * a.h_v;
  const int hk = h / (a.h_v / a.h_k);
  const int tid = threadIdx.x;
  const int j = tid >> 1, hh = tid & 1;
  const int row0 = hh * (G::NG / 2);  // first row group of this thread's half
  const bool kda = a.gate_kind != 0;
  const int slot = a.slots ? a.slots[b] : b;
  int len = a.lengths ? a.lengths[b] : a.L;
  len = len < 0 ? 0 : (len > a.L ? a.L : len);
  uint32_t st = 0;

  const int nchunks = (len + M::TC - 1) / M::TC;
  if (len > 0) prefill_fetch<D>(a, b, h, hk, 0, min(M::TC, len), tok);

  // S2[r][x] holds rows r NG + row0 + 2x and + 1 of column j
  float2 S2[G::RPT][NQ];
  if (a.S0) {
    const float* Sh = a.S0 + ((size_t)b * a.h_v + h) * D * D + j;
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int x = 0; x < NQ; ++x) {
        const int i = r * G::NG + row0 + 2 * x;
        S2[r][x] = make_float2(Sh[(size_t)i * D], Sh[(size_t)(i + 1) * D]);
      }
  } else {
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int x = 0; x < NQ; ++x) S2[r][x] = make_float2(0.f, 0.f);
  }
  cp_async_wait_all();
  __syncthreads();

  for (int c = 0; c < nchunks; ++c) {
    const float* cb = tok + (c & 1) * M::CHUNK;
    const int t0 = c * M::TC;
    const int n = min(M::TC, len - t0);
    if (c + 1 < nchunks)
      prefill_fetch<D>(a, b, h, hk, t0 + M::TC, min(M::TC, len - t0 - M::TC), tok + ((c + 1) & 1) * M::CHUNK);
    for (int u = 0; u < n; ++u) {
      const float* tk = cb + u * M::TOK;
      // gate
      if (!kda) {
        const float2 g2 = f2(tk[4 * D + 1]);
#pragma unroll
        for (int r = 0; r < G::RPT; ++r)
#pragma unroll
          for (int x = 0; x < NQ; ++x) S2[r][x] = __fmul2_rn(S2[r][x], g2);
      } else {
#pragma unroll
        for (int r = 0; r < G::RPT; ++r)
#pragma unroll
          for (int x = 0; x < NQ; x += 2) {
            const float4 gv = lds128(tk + 3 * D + r * G::NG + row0 + 2 * x);
            S2[r][x] = __fmul2_rn(S2[r][x], make_float2(gv.x, gv.y));
            S2[r][x + 1] = __fmul2_rn(S2[r][x + 1], make_float2(gv.z, gv.w));
          }
      }
      // S^T k, w = beta (v - P)
      const float P = column_tree<D>(S2, tk, hh);
      const float w = __fmul_rn(tk[4 * D], __fsub_rn(tk[2 * D + j], P));
      // delta update
      const float2 w2 = f2(w);
#pragma unroll
      for (int r = 0; r < G::RPT; ++r)
#pragma unroll
        for (int x = 0; x < NQ; x += 2) {
          const float4 kv = lds128(tk + r * G::NG + row0 + 2 * x);
          S2[r][x] = __ffma2_rn(make_float2(kv.x, kv.y), w2, S2[r][x]);
          S2[r][x + 1] = __ffma2_rn(make_float2(kv.z, kv.w), w2, S2[r][x + 1]);
        }
      // S^T q of the updated state
      const float O = column_tree<D>(S2, tk + D, hh);
      if (hh == 0) {
        if (O != O) st |= ST_NAN;
        a.o[(((size_t)b * a.L + t0 + u) * a.h_v + h) * D + j] = O;
      }
    }
    cp_async_wait_all();  // the next chunk's vectors, visible to all after the barrier
    __syncthreads();
  }

  // the final state: fp32 outputs straight from the registers, and the
  // row-major copy in shared memory that the quantization reads
  float* Ssh = reinterpret_cast<float*>(smem);
  const bool to_pool = slot >= 0 && slot < a.n_slots;
  if (!to_pool) st |= ST_SLOT;
  float* S_pool = (to_pool && a.fmt_fp32)
                      ? reinterpret_cast<float*>(a.pool) + ((size_t)slot * a.h_v + h) * D * D : nullptr;
  float* S_out = a.S_out ? a.S_out + ((size_t)b * a.h_v + h) * D * D : nullptr;
#pragma unroll
  for (int r = 0; r < G::RPT; ++r)
#pragma unroll
    for (int x = 0; x < NQ; ++x) {
      const int i = r * G::NG + row0 + 2 * x;
      if (S_out) {
        S_out[(size_t)i * D + j] = S2[r][x].x;
        S_out[(size_t)(i + 1) * D + j] = S2[r][x].y;
      }
      if (S_pool) {
        S_pool[(size_t)i * D + j] = S2[r][x].x;
        S_pool[(size_t)(i + 1) * D + j] = S2[r][x].y;
      }
      Ssh[i * D + j] = S2[r][x].x;
      Ssh[(i + 1) * D + j] = S2[r][x].y;
    }
  if (to_pool && !a.fmt_fp32) {
    // quantize once: T = S / c (as S * fl(1/c)), then the step kernels'
    // requantization in their thread map
    uint8_t* rec = smem + M::REGION;
    const uint32_t rb = a.t.rec_bytes[h];
    uint16_t* row_off = reinterpret_cast<uint16_t*>(rec + (rb + 15) / 16 * 16);
    uint8_t* row_code = reinterpret_cast<uint8_t*>(row_off + D);
    float* phi = reinterpret_cast<float*>(row_code + D);
    for (int i = tid; i < D; i += G::NT) {
      row_off[i] = a.t.row_off[(size_t)h * D + i];
      row_code[i] = a.t.row_code[(size_t)h * D + i];
      phi[i] = a.t.phi[(size_t)h * D + i];
    }
    for (uint32_t x = tid * 16; x < rb; x += G::NT * 16) *reinterpret_cast<uint4*>(rec + x) = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const int lane = tid & 31, warp = tid >> 5;
    const int cc = lane % G::LPR;
    const int rg = warp * G::RPW + lane / G::LPR;
    float2 T[G::RPT][8];
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      const float4* src = reinterpret_cast<const float4*>(Ssh + (size_t)(r * G::NG + rg) * D + 16 * cc);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 x = src[p];
        const float2 ic0 = make_float2(a.t.icol[(size_t)h * D + 16 * cc + 4 * p], a.t.icol[(size_t)h * D + 16 * cc + 4 * p + 1]);
        const float2 ic1 = make_float2(a.t.icol[(size_t)h * D + 16 * cc + 4 * p + 2], a.t.icol[(size_t)h * D + 16 * cc + 4 * p + 3]);
        T[r][2 * p] = __fmul2_rn(make_float2(x.x, x.y), ic0);
        T[r][2 * p + 1] = __fmul2_rn(make_float2(x.z, x.w), ic1);
      }
    }
    st |= requant_rows<D, 0>(rec, row_off, row_code, phi, rg, cc, false, T);
    __syncthreads();
    uint8_t* dst = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[h];
    for (uint32_t x = tid * 16; x < rb; x += G::NT * 16)
      *reinterpret_cast<uint4*>(dst + x) = *reinterpret_cast<const uint4*>(rec + x);
  }
  if (st) atomicOr(a.t.status, st);
}

}  // namespace sqk
