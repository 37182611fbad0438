// sq_prefill.cuh -- prefill handoff: the gated delta rule run over a whole
// prompt with the state held on chip, then quantized once into the pool.
//
// One CTA per (request, value head) tile. The fp32 state lives in registers
// (the thread map of the step kernels: a thread owns 16 value columns of RPT
// key rows) for every token of the prompt; each token applies exactly the
// arithmetic of the FP32 decode step (gate, S^T k column sums, delta update,
// S^T q column sums, same summation order), so a prefill of L tokens equals
// L FP32 decode steps bit for bit. The next token's vectors are fetched with
// cp.async into a second buffer while the current token is computed. After
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

// Shared memory of one prefill CTA: two token buffers, the two column-sum
// buffers and w; after the prompt, the record and the head's row tables
// reuse the column-sum region.
template <int D>
struct PrefillSmem {
  static constexpr int TOK = 4 * D + 8;                     // floats per token buffer: k q v g | beta g0 pad
  static constexpr int RED = Geo<D>::NG * D;                // floats per column-sum buffer
  static constexpr size_t TOK_BYTES = 2 * TOK * 4;
  static constexpr size_t RED_OFF = (TOK_BYTES + 127) / 128 * 128;
  static constexpr size_t W_OFF = RED_OFF + 2 * RED * 4;
  static constexpr size_t FIXED = W_OFF + D * 4;
  // record region (at RED_OFF): record, then row_off u16 [D], row_code u8 [D], phi f32 [D]
  static size_t bytes(uint32_t rec_cap) {
    const size_t rec = RED_OFF + (rec_cap + 15) / 16 * 16 + 2 * D + D + 4 * D;
    return rec > FIXED ? rec : FIXED;
  }
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Thread tid < D + 2 fetches one piece of token t's inputs into `buf`:
// 16-byte chunks of k, q, v (and g per key channel), then beta and the
// per-head gate.
template <int D>
__device__ __forceinline__ void prefill_fetch(const PrefillArgs& a, int b, int h, int hk, int t, float* buf) {
  const int tid = threadIdx.x;
  const size_t bt = (size_t)b * a.L + t;
  constexpr int C = D / 4;
  if (tid < C) {
    cp_async16(buf + 4 * tid, a.k + (bt * a.h_k + hk) * D + 4 * tid);
  } else if (tid < 2 * C) {
    cp_async16(buf + D + 4 * (tid - C), a.q + (bt * a.h_k + hk) * D + 4 * (tid - C));
  } else if (tid < 3 * C) {
    cp_async16(buf + 2 * D + 4 * (tid - 2 * C), a.v + (bt * a.h_v + h) * D + 4 * (tid - 2 * C));
  } else if (tid < 4 * C) {
    if (a.gate_kind != 0) cp_async16(buf + 3 * D + 4 * (tid - 3 * C), a.g + (bt * a.h_v + h) * D + 4 * (tid - 3 * C));
  } else if (tid == 4 * C) {
    cp_async4(buf + 4 * D, a.beta + bt * a.h_v + h);
  } else if (tid == 4 * C + 1) {
    if (a.gate_kind == 0) cp_async4(buf + 4 * D + 1, a.g + bt * a.h_v + h);
  }
  cp_async_commit();
}

template <int D>
__global__ void __launch_bounds__(Geo<D>::NT, 2) k_prefill(const PrefillArgs a) {
  using G = Geo<D>;
  using M = PrefillSmem<D>;
  static_assert(G::NT >= D + 2, "one fetching thread per 16-byte piece of a token");
  extern __shared__ __align__(128) uint8_t smem[];
  float* tok = reinterpret_cast<float*>(smem);
  float* redP = reinterpret_cast<float*>(smem + M::RED_OFF);
  float* redO = redP + M::RED;
  float* wsh = reinterpret_cast<float*>(smem + M::W_OFF);

  const int tile = blockIdx.x;
  const int b = tile / a.h_v;
  const int h = tile - b * a.h_v;
  const int hk = h / (a.h_v / a.h_k);
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int cc = lane % G::LPR;
  const int rg = warp * G::RPW + lane / G::LPR;
  const int slot = a.slots ? a.slots[b] : b;
  int len = a.lengths ? a.lengths[b] : a.L;
  len = len < 0 ? 0 : (len > a.L ? a.L : len);
  uint32_t st = 0;

  if (len > 0) prefill_fetch<D>(a, b, h, hk, 0, tok);

  float2 T[G::RPT][8];
  if (a.S0) {
    const float* Sh = a.S0 + ((size_t)b * a.h_v + h) * D * D;
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      const float4* src = reinterpret_cast<const float4*>(Sh + (size_t)(r * G::NG + rg) * D + 16 * cc);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 x = src[p];
        T[r][2 * p] = make_float2(x.x, x.y);
        T[r][2 * p + 1] = make_float2(x.z, x.w);
      }
    }
  } else {
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int p = 0; p < 8; ++p) T[r][p] = make_float2(0.f, 0.f);
  }
  cp_async_wait_all();
  __syncthreads();

  for (int t = 0; t < len; ++t) {
    const float* cur = tok + (t & 1) * M::TOK;
    if (t + 1 < len) prefill_fetch<D>(a, b, h, hk, t + 1, tok + ((t + 1) & 1) * M::TOK);
    const float beta = cur[4 * D];
    float kr[G::RPT], qr[G::RPT];
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      const int i = r * G::NG + rg;
      kr[r] = cur[i];
      qr[r] = cur[D + i];
      const float gr = a.gate_kind == 0 ? cur[4 * D + 1] : cur[3 * D + i];
#pragma unroll
      for (int p = 0; p < 8; ++p) T[r][p] = __fmul2_rn(T[r][p], f2(gr));
    }
    // S^T k of the gated state
    float2 part[8];
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int p = 0; p < 8; ++p)
        part[p] = r == 0 ? __fmul2_rn(T[r][p], f2(kr[r])) : __ffma2_rn(T[r][p], f2(kr[r]), part[p]);
    column_deposit<D>(redP, rg, cc, part);
    __syncthreads();
    {
      const float P = column_total<D>(redP);
      if ((tid & 1) == 0) {
        const int j = tid >> 1;
        wsh[j] = __fmul_rn(beta, __fsub_rn(cur[2 * D + j], P));
      }
    }
    __syncthreads();
    float2 W[8];
    {
      const float4* wsrc = reinterpret_cast<const float4*>(wsh + 16 * cc);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 x = wsrc[p];
        W[2 * p] = make_float2(x.x, x.y);
        W[2 * p + 1] = make_float2(x.z, x.w);
      }
    }
    // delta update and S^T q of the updated state
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        T[r][p] = __ffma2_rn(f2(kr[r]), W[p], T[r][p]);
        part[p] = r == 0 ? __fmul2_rn(T[r][p], f2(qr[r])) : __ffma2_rn(T[r][p], f2(qr[r]), part[p]);
      }
    column_deposit<D>(redO, rg, cc, part);
    cp_async_wait_all();  // the next token's inputs, visible to all after the barrier
    __syncthreads();
    {
      const float O = column_total<D>(redO);
      if ((tid & 1) == 0) {
        const int j = tid >> 1;
        if (O != O) st |= ST_NAN;
        a.o[(((size_t)b * a.L + t) * a.h_v + h) * D + j] = O;
      }
    }
  }

  if (a.S_out) {
    float* Sh = a.S_out + ((size_t)b * a.h_v + h) * D * D;
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      float4* dst = reinterpret_cast<float4*>(Sh + (size_t)(r * G::NG + rg) * D + 16 * cc);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        dst[p] = make_float4(T[r][2 * p].x, T[r][2 * p].y, T[r][2 * p + 1].x, T[r][2 * p + 1].y);
    }
  }

  if (slot < 0 || slot >= a.n_slots) {
    st |= ST_SLOT;
  } else if (a.fmt_fp32) {
    float* Sh = reinterpret_cast<float*>(a.pool) + ((size_t)slot * a.h_v + h) * D * D;
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      float4* dst = reinterpret_cast<float4*>(Sh + (size_t)(r * G::NG + rg) * D + 16 * cc);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        dst[p] = make_float4(T[r][2 * p].x, T[r][2 * p].y, T[r][2 * p + 1].x, T[r][2 * p + 1].y);
    }
  } else {
    // quantize once: T = S / c (as S * fl(1/c)), then the step kernels' requantization
    __syncthreads();  // every thread is done with the column-sum buffers
    uint8_t* rec = smem + M::RED_OFF;
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
    float2 ic[8];
#pragma unroll
    for (int p = 0; p < 8; ++p)
      ic[p] = make_float2(a.t.icol[(size_t)h * D + 16 * cc + 2 * p], a.t.icol[(size_t)h * D + 16 * cc + 2 * p + 1]);
#pragma unroll
    for (int r = 0; r < G::RPT; ++r)
#pragma unroll
      for (int p = 0; p < 8; ++p) T[r][p] = __fmul2_rn(T[r][p], ic[p]);
    __syncthreads();
    st |= requant_rows<D, 0>(rec, row_off, row_code, phi, rg, cc, false, T);
    __syncthreads();
    uint8_t* dst = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[h];
    for (uint32_t x = tid * 16; x < rb; x += G::NT * 16)
      *reinterpret_cast<uint4*>(dst + x) = *reinterpret_cast<const uint4*>(rec + x);
  }
  if (st) atomicOr(a.t.status, st);
}

}  // namespace sqk
