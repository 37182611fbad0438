// sq_kernels.cuh -- sm_100a building blocks of the quantized-state decode
// step, and the kernels around it.
//
// The FP32-state baseline step is persistent like the packed step: one CTA
// owns one (request, value head) tile at a time, the tile (plus its small
// vectors) arrives in shared memory through 1-D TMA bulk copies
// (cp.async.bulk, no multicast) completed on an mbarrier, NSTAGE tiles ahead
// of the one being computed, and goes back in place with a bulk store.
// Thread map of the kernels in this file (Geo): a thread owns 16
// consecutive value columns of RPT key rows (d = 128: 256 threads, 4 rows
// each; 8 lanes cover one row, so a row's 16-column chunk is 2*b bytes =
// b/2 whole 32-bit words for every width b). Column sums go through shared
// memory; row maxima use warp shuffles over the lanes of a row.
//
// The fused packed step itself is in sq_step.cuh; this file holds the code
// formats (bit-field unpacking and packing, fp16 pivots), the shared
// requantization helpers, the FP32-state baseline step and the quantize /
// dequantize kernels. Every elementwise operation is an explicit
// round-to-nearest intrinsic (the library is built with --fmad=false), so
// codes are reproducible.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sqk {

constexpr uint32_t ST_NAN = 1u;
constexpr uint32_t ST_SAT = 2u;
constexpr uint32_t ST_SLOT = 4u;
constexpr uint32_t ST_TIMEOUT = 8u;
constexpr uint8_t ROW_PIVOT = 16;  // row_code value of an FP16 pivot row

// Device tables owned by a handle (one allocation, see sq_api.cu).
struct Tables {
  const uint32_t* rec_off;    // [h_v] byte offset of head h's record inside a slot
  const uint32_t* rec_bytes;  // [h_v] record size (multiple of 16)
  const uint16_t* row_off;    // [h_v*d] byte offset of key row i inside the record
  const uint8_t* row_code;    // [h_v*d] 2, 4, 6, 8 or ROW_PIVOT
  const uint8_t* row_perm;    // [h_v*d] packed step: row held in thread slot s (mixed-width heads: rows
                              //         grouped by width, so a warp's rows share a width); else s
  const float* col;           // [h_v*d] c_j
  const float* icol;          // [h_v*d] fl(1 / c_j)
  const float* phi;           // [h_v*d] phi_i
  const uint8_t* head_kind;   // [h_v] width shared by all rows of the head (ROW_PIVOT: all pivot), 0: mixed
  uint32_t* status;           // device status word
  uint32_t* sched;            // packed step: [0] next chunk of tiles, [1] CTAs done (both 0 between launches)
  uint32_t* xcount;           // packed step: columns whose S^T k was summed exactly (running count)
};

struct StepArgs {
  uint8_t* pool;        // packed pool, or fp32 S pool for the FP32 kernel
  const float* q;       // [B, h_k, d]
  const float* k;       // [B, h_k, d]
  const float* v;       // [B, h_v, d]
  const float* beta;    // [B, h_v]
  const float* g;       // [B, h_v] or [B, h_v, d]
  float* o;             // [B, h_v, d]
  const int32_t* slots; // [B] or null
  int32_t B, h_v, h_k, n_slots, gate_kind;
  int32_t nstage;
  int32_t chunk;        // packed step: tiles per scheduling chunk
  uint32_t rec_cap;     // bytes reserved for a record in a stage (multiple of 128)
  uint32_t stage_bytes; // rec_cap + aux bytes, multiple of 128
  uint64_t slot_bytes;
  uint64_t wait_ns;     // limit of every bounded wait inside the kernel
  uint32_t test_extra_tx;  // testing only: extra bytes the stage of tile (request 0, head 0) expects (0: none)
  Tables t;
};

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after ~max_ns nanoseconds of global timer time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t max_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 > max_ns) return false;
  }
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// max that propagates NaN
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// ---------------------------------------------------------- tile geometry
template <int D>
struct Geo {
  static constexpr int LPR = D / 16;          // lanes per key row (16 columns each)
  static constexpr int RPW = 32 / LPR;        // rows a warp covers per pass
  static constexpr int NW = D == 128 ? 8 : (D == 64 ? 4 : 2);
  static constexpr int NT = 32 * NW;          // threads per CTA
  static constexpr int NG = NW * RPW;         // row groups (= rows per pass of the CTA)
  static constexpr int RPT = D / NG;          // rows per thread
  static constexpr int AUX = (32 * D + 32 + 127) / 128 * 128;  // vector bytes per stage (see stage layout)
  static_assert(RPT >= 1 && RPT * NG == D, "bad geometry");
};

// Stage layout: [k f32 D][q f32 D][v f32 D][g f32 D][c f32 D][ic f32 D]
//               [phi f32 D][row_off u16 D][row_code u8 D][row_perm u8 D]
//               [TileHdr 32 B] (padded to Geo<D>::AUX bytes) [record: rec_cap]
// Every offset but the stage's own base is a compile-time constant.
template <int D>
struct Stage {
  uint8_t* base;
  uint32_t rec_cap;
  __device__ float* k() const { return reinterpret_cast<float*>(base); }
  __device__ float* q() const { return k() + D; }
  __device__ float* v() const { return k() + 2 * D; }
  __device__ float* g() const { return k() + 3 * D; }
  __device__ float* c() const { return k() + 4 * D; }
  __device__ float* ic() const { return k() + 5 * D; }
  __device__ float* phi() const { return k() + 6 * D; }
  __device__ uint16_t* row_off() const { return reinterpret_cast<uint16_t*>(k() + 7 * D); }
  __device__ uint8_t* row_code() const { return reinterpret_cast<uint8_t*>(row_off() + D); }
  __device__ uint8_t* row_perm() const { return row_code() + D; }
  __device__ struct TileHdr* hdr() const { return reinterpret_cast<struct TileHdr*>(row_perm() + D); }
  __device__ uint8_t* rec() const { return base + Geo<D>::AUX; }
};

// Per-tile scalars the producing thread writes next to the stage's data
// before the stage's mbarrier completes (so consumers never wait on global
// memory for them).
struct TileHdr {
  uint8_t* dst;     // global address of the record (store target)
  uint32_t bytes;   // record bytes
  int32_t valid;    // 0: slot id out of range, nothing was loaded
  float beta;
  float g;          // the head's gate (GDN); unused for KDA
  int32_t kind;     // width shared by every row of the head (ROW_PIVOT: all pivot), 0: mixed
  int32_t tile;     // packed step: b * h_v + h of the tile in this stage, or -1: no more tiles
};

// ------------------------------------------------------- code unpacking
// Field j (b bits) of a 16-code chunk held in b/2 words, as the float
// 2^23 + field (exact): OR the field into the exponent pattern of 2^23.
template <int B>
__device__ __forceinline__ uint32_t field_as_magic(const uint32_t* w, int j) {
  const int bit = B * j;
  const int wi = bit >> 5;
  const int sh = bit & 31;
  uint32_t x;
  if (sh + B <= 32)
    x = w[wi] >> sh;
  else
    x = __funnelshift_r(w[wi], w[wi + 1], sh);
  return 0x4B000000u | (x & ((1u << B) - 1u));
}

// 16 codes of width B -> float values q (exact), as 8 float2 pairs.
template <int B>
__device__ __forceinline__ void unpack16(const uint32_t* w, float2 (&f)[8]) {
  const float off = 8388608.0f + (float)(1 << (B - 1));
  const float2 offv = make_float2(-off, -off);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float2 m = make_float2(__uint_as_float(field_as_magic<B>(w, 2 * p)),
                           __uint_as_float(field_as_magic<B>(w, 2 * p + 1)));
    f[p] = __fadd2_rn(m, offv);
  }
}

// fp64 view of a b-bit field f for the S^T k column sum: the field is placed
// at bits [20-E, 20-E+b) of a high word whose exponent field is 1023 + E, so
// that this word over a zero low word is the double 2^E + f exactly. 8-bit
// fields go to a byte boundary (E = 12), where one byte permute places them;
// the other widths use E = b.
//
// Read as a float, the same word is v = 2^EF (1 + M0 2^-23) + f 2^(POS+EF-23)
// (EF, M0: exponent and mantissa of the float view of EXP), so the code
// q = f - 2^(b-1) is exactly fma(v, K, -C) with K = 2^(23-POS-EF) and
// C = 2^(23-POS) + (M0 >> POS) + 2^(b-1), where M0 >> POS = ((1023+E) & 7) 2^E.
template <int B>
struct FieldPos {
  static constexpr int E = B == 8 ? 12 : B;
  static constexpr int POS = 20 - E;
  static constexpr uint32_t EXP = (0x3FFu + (uint32_t)E) << 20;
  static constexpr int EF = (int)((EXP >> 23) & 0xFFu) - 127;
  static constexpr float K = (float)(1u << (23 - POS - EF));
  static constexpr float C = (float)((1u << (23 - POS)) + ((0x3FFu + (uint32_t)E) & 7u) * (1u << E) + (1u << (B - 1)));
};

// Field j of a 16-code chunk held in b/2 words, in place as described above.
template <int B>
__device__ __forceinline__ uint32_t field_hi(const uint32_t* w, int j) {
  constexpr int POS = FieldPos<B>::POS;
  constexpr uint32_t EXP = FieldPos<B>::EXP;
  if constexpr (B == 8) {
    return __byte_perm(w[j >> 2], EXP, 0x7604u | ((uint32_t)(j & 3) << 4));
  } else {
    constexpr uint32_t MASK = ((1u << B) - 1u) << POS;
    const int bit = B * j;
    const int wi = bit >> 5;
    const int sh = bit & 31;
    uint32_t x;
    if (sh + B <= 32)
      x = sh >= POS ? (w[wi] >> (sh - POS)) : (w[wi] << (POS - sh));
    else
      x = __funnelshift_r(w[wi], w[wi + 1], sh - POS);  // a straddling field always has sh > POS
    return EXP | (x & MASK);
  }
}

// Per-row constant of the fp64 column sum: a row of width b adds
// (2^E + f) kap to every column, so (2^E + 2^(b-1)) kap is taken off once
// per row to leave q kap (f = q + 2^(b-1)).
__device__ __forceinline__ double code_offset(int code) {
  const int E = code == 8 ? 12 : code;
  return (double)((1 << E) + (1 << (code - 1)));
}

// The b/2 code words (quantized row, b in {2,4,6,8}) or 8 fp16-pair words
// (pivot row) of the 16-column chunk cc of one row, from shared memory or,
// for GLOBAL, from the pool itself. VEC: the chunk is aligned to its size
// (up to 16 bytes), true for every row of a head of uniform width; rows of
// mixed-width heads are only 4-byte aligned (d = 32: a 6-bit row is 24 B).
template <int B, bool GLOBAL, bool VEC = true>
__device__ __forceinline__ void chunk_words(const uint8_t* row, int cc, uint32_t (&w)[B / 2]) {
  const uint8_t* p = row + 2 * B * cc;
  if constexpr (!VEC) {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  } else if constexpr (GLOBAL) {
    static_assert(B % 8 == 0, "global rows are read in 16-byte pieces");
#pragma unroll
    for (int q = 0; q < B / 8; ++q) {
      uint4 x;
      asm("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                   : "l"(p + 16 * q));
      w[4 * q] = x.x; w[4 * q + 1] = x.y; w[4 * q + 2] = x.z; w[4 * q + 3] = x.w;
    }
  } else if constexpr (B == 8 || B == 16) {
#pragma unroll
    for (int q = 0; q < B / 8; ++q) {
      const uint4 x = reinterpret_cast<const uint4*>(p)[q];
      w[4 * q] = x.x; w[4 * q + 1] = x.y; w[4 * q + 2] = x.z; w[4 * q + 3] = x.w;
    }
  } else if constexpr (B == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x; w[1] = x.y;
  } else {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
}

// Constant part of packed word `wi` when every fb[j] = 0x4B000000 + field_j
// is shifted into place (see pack16).
template <int B>
__host__ __device__ constexpr uint32_t pack_const(int wi) {
  uint32_t c = 0;
  for (int j = 0; j < 16; ++j) {
    const int lo = B * j - 32 * wi;
    if (lo >= 32 || lo + B <= 0) continue;
    c += lo >= 0 ? (0x4B000000u << lo) : (0x4B000000u >> (-lo));
  }
  return c;
}

// Pack 16 magic-number floats fb[j] = bits(2^23 + field_j) into b/2 words.
// 8-bit: byte permutes. Otherwise: the fields occupy disjoint bits and the
// constant 0x4B000000 is a multiple of 2^24 (so shifting it right by less
// than 24 never mixes with a field), hence each word is the sum of the
// shifted fb[j] minus the same sum of shifted constants (mod 2^32): one
// multiply-add per field.
template <int B>
__device__ __forceinline__ void pack16(const uint32_t (&fb)[16], uint32_t* w) {
  if constexpr (B == 8) {
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t lo = __byte_perm(fb[4 * wi], fb[4 * wi + 1], 0x0040);
      const uint32_t hi = __byte_perm(fb[4 * wi + 2], fb[4 * wi + 3], 0x0040);
      w[wi] = __byte_perm(lo, hi, 0x5410);
    }
  } else {
#pragma unroll
    for (int wi = 0; wi < B / 2; ++wi) {
      uint32_t acc = 0u - pack_const<B>(wi);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int lo = B * j - 32 * wi;
        if (lo >= 32 || lo + B <= 0) continue;
        if (lo >= 0)
          acc += fb[j] * (1u << lo);
        else
          acc += fb[j] >> (-lo);
      }
      w[wi] = acc;
    }
  }
}

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// Load the 16-column chunk of one row (as column-normalised values times
// `mul`) from a record in shared memory: quantized row -> q * mul;
// pivot row -> fp16 value * mul.
template <int B>
__device__ __forceinline__ void load_row_q(const uint8_t* row, int cc, float mul, float2 (&t)[8]) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 2 * B * cc);
  uint32_t w[B / 2];
#pragma unroll
  for (int i = 0; i < B / 2; ++i) w[i] = src[i];
  float2 f[8];
  unpack16<B>(w, f);
#pragma unroll
  for (int p = 0; p < 8; ++p) t[p] = __fmul2_rn(f[p], f2(mul));
}

__device__ __forceinline__ void load_row_pivot(const uint8_t* row, int cc, float mul, float2 (&t)[8]) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 32 * cc);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    __half2 h2 = *reinterpret_cast<const __half2*>(src + p);
    float2 x = __half22float2(h2);
    t[p] = __fmul2_rn(x, f2(mul));
  }
}

// Dispatch on the row code.
__device__ __forceinline__ void load_row(const uint8_t* row, uint8_t code, int cc, float mul, float2 (&t)[8]) {
  switch (code) {
    case 8: load_row_q<8>(row, cc, mul, t); break;
    case 6: load_row_q<6>(row, cc, mul, t); break;
    case 4: load_row_q<4>(row, cc, mul, t); break;
    case 2: load_row_q<2>(row, cc, mul, t); break;
    default: load_row_pivot(row, cc, mul, t); break;
  }
}

// sign(x) min(|x|, lim) for lim >= 0 (one instruction on sm_100).
__device__ __forceinline__ float clamp_abs(float x, float lim) {
  float r;
  asm("min.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(x), "f"(lim));
  return r;
}

// Requantize one row chunk of T' with inverse scale `ir` = fl(1 / r') and
// write it back. The code is the nearest integer (ties to even) to the exact
// product T' * ir, clamped to [-qmax, qmax]. The clamp is applied to T'
// first, at lim = qmax r' (exact in fp32): a |T'| above lim gives a product
// of at least lim * ir = qmax (1 + e), |e| <= 2^-24, whose nearest integer
// is qmax, and lim itself gives exactly qmax, so clamping T' to lim and
// rounding equals rounding and clamping the code. fma(T'c, ir, 2^23 +
// 2^(b-1)) then rounds the exact product to the nearest integer in the
// window [2^23, 2^24) where floats are integers, and its low b bits are the
// stored field.
template <int B>
__device__ __forceinline__ void store_row_q(uint8_t* row, int cc, float ir, float lim, const float2 (&t)[8]) {
  const float magic = 8388608.0f + (float)(1 << (B - 1));
  uint32_t fb[16];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 tc = make_float2(clamp_abs(t[p].x, lim), clamp_abs(t[p].y, lim));
    const float2 n = __ffma2_rn(tc, f2(ir), f2(magic));
    fb[2 * p] = __float_as_uint(n.x);
    fb[2 * p + 1] = __float_as_uint(n.y);
  }
  uint32_t w[B / 2];
  pack16<B>(fb, w);
  uint32_t* dst = reinterpret_cast<uint32_t*>(row + 2 * B * cc);
#pragma unroll
  for (int i = 0; i < B / 2; ++i) dst[i] = w[i];
}

__device__ __forceinline__ void store_row_zero(uint8_t* row, int B, int cc) {
  // all codes 0: every field is 2^(b-1) (given to pack16 in its 2^23 + field form)
  uint32_t fb[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) fb[j] = 0x4B000000u | (1u << (B - 1));
  uint32_t* dst = reinterpret_cast<uint32_t*>(row + 2 * B * cc);
  switch (B) {
    case 8: { uint32_t w[4]; pack16<8>(fb, w); for (int i = 0; i < 4; ++i) dst[i] = w[i]; } break;
    case 6: { uint32_t w[3]; pack16<6>(fb, w); for (int i = 0; i < 3; ++i) dst[i] = w[i]; } break;
    case 4: { uint32_t w[2]; pack16<4>(fb, w); for (int i = 0; i < 2; ++i) dst[i] = w[i]; } break;
    default: { uint32_t w[1]; pack16<2>(fb, w); dst[0] = w[0]; } break;
  }
}

// fp16 pivot row: RNE with saturation at +-65504; NaN stores 0. GLOBAL: the
// row is in the pool (16-byte aligned chunks), else in shared memory.
template <bool GLOBAL>
__device__ __forceinline__ uint32_t store_row_pivot(uint8_t* row, int cc, const float2 (&t)[8]) {
  uint32_t st = 0;
  uint32_t w[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float x0 = t[p].x, x1 = t[p].y;
    if (x0 != x0) { x0 = 0.0f; st |= ST_NAN; }
    if (x1 != x1) { x1 = 0.0f; st |= ST_NAN; }
    if (fabsf(x0) > 65504.0f) { x0 = copysignf(65504.0f, x0); st |= ST_SAT; }
    if (fabsf(x1) > 65504.0f) { x1 = copysignf(65504.0f, x1); st |= ST_SAT; }
    __half2 h = __floats2half2_rn(x0, x1);
    w[p] = *reinterpret_cast<uint32_t*>(&h);
  }
  uint8_t* dst = row + 32 * cc;
  if constexpr (GLOBAL) {
#pragma unroll
    for (int q = 0; q < 2; ++q)
      asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 16 * q), "r"(w[4 * q]),
                   "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                   : "memory");
  } else {
#pragma unroll
    for (int p = 0; p < 8; ++p) reinterpret_cast<uint32_t*>(dst)[p] = w[p];
  }
  return st;
}

// Byte offset of key row i inside a head record: from the per-head table,
// or, when every row of the head has width KC (KC = ROW_PIVOT for an
// all-pivot head), from the closed form 2d + i * row_bytes.
template <int D, int KC>
__device__ __forceinline__ uint32_t row_offset(const uint16_t* row_off, int i) {
  if constexpr (KC == 0) {
    return row_off[i];
  } else {
    constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
    return 2u * D + (uint32_t)i * rb;
  }
}

// Requantization of the RPT rows a thread holds: row maxima across the LPR
// lanes of each row, one row scale per row (computed by one lane of the row
// and handed to the others by shuffle), codes; writes the record in shared
// memory. `finite`: the tile's inputs were all finite, so no T' is NaN and
// the plain maximum equals the NaN-propagating one. Returns status bits.
template <int D, int KC>
__device__ __forceinline__ uint32_t requant_rows(uint8_t* rec, const uint16_t* row_off, const uint8_t* row_code,
                                                 const float* phi, int rg, int cc, bool finite,
                                                 float2 (&T)[Geo<D>::RPT][8]) {
  using G = Geo<D>;
  (void)row_off;
  uint32_t st = 0;
  float m[G::RPT];
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    float x = 0.0f;
    if (finite) {
#pragma unroll
      for (int p = 0; p < 8; ++p) x = fmaxf(x, fmaxf(fabsf(T[r][p].x), fabsf(T[r][p].y)));
#pragma unroll
      for (int s = 1; s < G::LPR; s <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, s));
    } else {
#pragma unroll
      for (int p = 0; p < 8; ++p) x = fmax_nan(x, fmax_nan(fabsf(T[r][p].x), fabsf(T[r][p].y)));
#pragma unroll
      for (int s = 1; s < G::LPR; s <<= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, s));
    }
    m[r] = x;
  }
  // lane cc of a row group computes the scale of row slot cc % RPT
  const int mine = cc % G::RPT;
  float mm = m[0];
#pragma unroll
  for (int r = 1; r < G::RPT; ++r) mm = mine == r ? m[r] : mm;
  const int im = mine * G::NG + rg;
  const int cm = KC ? KC : row_code[im];
  float ir_m = 0.0f, lim_m = 0.0f;
  uint16_t rbits = 0x3C00;  // pivot rows keep fp16 1.0 in their scale slot
  if (cm != ROW_PIVOT) {
    if (mm != mm) {
      rbits = 0;
      st |= ST_NAN;
    } else {
      const float qm = (float)((1 << (cm - 1)) - 1);
      const float s = __fdiv_rn(__fmul_rn(phi[im], mm), qm);
      __half rh;
      if (s > 65504.0f) {
        rh = __ushort_as_half((unsigned short)0x7BFF);
        st |= ST_SAT;
      } else {
        rh = __float2half_ru(s);
      }
      const float R = __half2float(rh);
      ir_m = (R == 0.0f) ? 0.0f : __frcp_rn(R);
      lim_m = __fmul_rn((float)((1 << (cm - 1)) - 1), R);  // qmax r', exact
      rbits = __half_as_ushort(rh);
    }
  }
  if (cc < G::RPT) reinterpret_cast<uint16_t*>(rec)[im] = rbits;
  const int lane = threadIdx.x & 31;
  const int base = lane - cc;
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const float ir = __shfl_sync(0xffffffffu, ir_m, base + r);
    const float lim = __shfl_sync(0xffffffffu, lim_m, base + r);
    const int i = r * G::NG + rg;
    const int code = KC ? KC : row_code[i];
    uint8_t* row = rec + row_offset<D, KC>(row_off, i);
    if (code == ROW_PIVOT) {
      st |= store_row_pivot<false>(row, cc, T[r]);
    } else if (m[r] != m[r]) {  // a NaN in the row: scale 0, all codes 0
      store_row_zero(row, code, cc);
    } else {
      switch (code) {
        case 8: store_row_q<8>(row, cc, ir, lim, T[r]); break;
        case 6: store_row_q<6>(row, cc, ir, lim, T[r]); break;
        case 4: store_row_q<4>(row, cc, ir, lim, T[r]); break;
        default: store_row_q<2>(row, cc, ir, lim, T[r]); break;
      }
    }
  }
  return st;
}

// Column sums. Every thread deposits its 16 partials for its row group;
// a thread's chunks are stored rotated by its column block (XOR swizzle) so
// the eight lanes of a row write eight different bank groups. Then two
// adjacent threads own one column (thread 2j and 2j+1 each add half of the
// row groups) and combine with one shuffle; column = threadIdx.x >> 1.
template <int D>
__device__ __forceinline__ void column_deposit(float* red, int rg, int cc, const float2 (&part)[8]) {
  const int sw = (cc >> 1) & 3;
#pragma unroll
  for (int p = 0; p < 4; ++p)
    *reinterpret_cast<float4*>(red + rg * D + 16 * cc + 4 * (p ^ sw)) =
        make_float4(part[2 * p].x, part[2 * p].y, part[2 * p + 1].x, part[2 * p + 1].y);
}

template <int D>
__device__ __forceinline__ float column_total(const float* red) {
  using G = Geo<D>;
  static_assert(G::NT == 2 * D, "two threads per column");
  const int j = threadIdx.x >> 1;
  const int hh = threadIdx.x & 1;
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 4 * ((e >> 2) ^ ((cj >> 1) & 3)) + (e & 3);
  // four independent partial sums keep the dependent chains short
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < G::NG / 2; ++g) a[g & 3] = __fadd_rn(a[g & 3], red[(hh * (G::NG / 2) + g) * D + off]);
  const float t = __fadd_rn(__fadd_rn(a[0], a[1]), __fadd_rn(a[2], a[3]));
  return __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 1));
}

// Deposit, barrier, total. The caller syncs before reusing `red`.
template <int D>
__device__ __forceinline__ float column_sum(float* red, int rg, int cc, const float2 (&part)[8]) {
  column_deposit<D>(red, rg, cc, part);
  __syncthreads();
  return column_total<D>(red);
}

// fp64 deposit of the 8 partials of half `half` of a thread's 16 columns
// (same swizzle idea: 16-byte chunks of two doubles rotated by cc).
template <int D>
__device__ __forceinline__ void deposit_f64(double* red, int rg, int cc, int half, const double (&acc)[8]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int chunk = 4 * half + p;
    *reinterpret_cast<double2*>(red + rg * D + 16 * cc + 2 * (chunk ^ (cc & 7))) =
        make_double2(acc[2 * p], acc[2 * p + 1]);
  }
}

// Column total of the fp64 partials, rounded once to fp32 (two threads per
// column as in column_total; column = threadIdx.x >> 1). The caller syncs
// after the deposits.
template <int D>
__device__ __forceinline__ float column_total_f64(const double* red) {
  using G = Geo<D>;
  const int j = threadIdx.x >> 1;
  const int hh = threadIdx.x & 1;
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 2 * ((e >> 1) ^ (cj & 7)) + (e & 1);
  double a[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int g = 0; g < G::NG / 2; ++g) a[g & 3] += red[(hh * (G::NG / 2) + g) * D + off];
  const double t = (a[0] + a[1]) + (a[2] + a[3]);
  return __double2float_rn(t + __shfl_xor_sync(0xffffffffu, t, 1));
}

// ================================================================ step kernels
// Scalars of one tile, loaded by the producing thread one tile ahead of the
// issue that needs them, so that their global-memory latency overlaps a
// whole tile of compute.
struct TileScalars {
  int tile;
  int b, h;
  int slot;
  uint32_t rec_off, rec_bytes;
  float beta, g;
  int kind;
};

template <int D>
__device__ __forceinline__ TileScalars load_scalars(const StepArgs& a, int tile, int t1, bool packed) {
  TileScalars x;
  x.tile = tile;
  if (tile >= t1) return x;
  x.b = tile / a.h_v;
  x.h = tile - x.b * a.h_v;
  x.slot = a.slots ? a.slots[x.b] : x.b;
  x.rec_off = packed ? a.t.rec_off[x.h] : 0u;
  x.rec_bytes = packed ? a.t.rec_bytes[x.h] : 4u * D * D;
  x.beta = a.beta[tile];
  x.g = a.gate_kind == 0 ? a.g[tile] : 0.0f;
  x.kind = packed ? a.t.head_kind[x.h] : 0;
  return x;
}

// ----------------------------------------------------------- FP32 state
// The unquantized baseline: fp32 S in the pool, the same update rule in
// fp32 (gate, S^T k, delta update, o), one tile per CTA iteration with the
// tile held in registers.
template <int D>
__device__ __forceinline__ void issue_fp32(const StepArgs& a, const TileScalars& x, uint8_t* stage_base,
                                           uint64_t* bar) {
  Stage<D> s{stage_base, a.rec_cap};
  TileHdr* hd = s.hdr();
  if (x.slot < 0 || x.slot >= a.n_slots) {
    hd->valid = 0;
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
    return;
  }
  const int b = x.b, h = x.h;
  const int hk = h / (a.h_v / a.h_k);
  const uint32_t vec = 4u * D;
  const bool kda = a.gate_kind != 0;
  uint8_t* rec_src = a.pool + ((uint64_t)x.slot * a.h_v + h) * (uint64_t)(4u * D * D);
  hd->dst = rec_src;
  hd->bytes = x.rec_bytes;
  hd->valid = 1;
  hd->beta = x.beta;
  hd->g = x.g;
  hd->kind = 0;
  const uint32_t tx = x.rec_bytes + 3 * vec + (kda ? vec : 0u);
  mbar_arrive_expect_tx(bar, tx);  // release: the header stores above become visible with the phase
  bulk_g2s(s.rec(), rec_src, x.rec_bytes, bar);
  bulk_g2s(s.k(), a.k + ((size_t)b * a.h_k + hk) * D, vec, bar);
  bulk_g2s(s.q(), a.q + ((size_t)b * a.h_k + hk) * D, vec, bar);
  bulk_g2s(s.v(), a.v + ((size_t)b * a.h_v + h) * D, vec, bar);
  if (kda) bulk_g2s(s.g(), a.g + ((size_t)b * a.h_v + h) * D, vec, bar);
}

template <int D>
__device__ __forceinline__ void tile_body_fp32(const StepArgs& a, const Stage<D>& S, const TileHdr& hd, float* red,
                                               float* wsh, float* o, int rg, int cc, uint32_t& st) {
  using G = Geo<D>;
  const int tid = threadIdx.x;
  const float* ks = S.k();
  const float* qs = S.q();
  float kr[G::RPT], qr[G::RPT], gr[G::RPT];
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const int i = r * G::NG + rg;
    kr[r] = ks[i];
    qr[r] = qs[i];
    gr[r] = a.gate_kind == 0 ? hd.g : S.g()[i];
  }
  // gate and column sum S^T k
  float2 T[G::RPT][8];
  float2 part[8];
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const int i = r * G::NG + rg;
    const float4* src = reinterpret_cast<const float4*>(S.rec() + ((size_t)i * D + 16 * cc) * 4);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float4 x = src[p];
      T[r][2 * p] = __fmul2_rn(make_float2(x.x, x.y), f2(gr[r]));
      T[r][2 * p + 1] = __fmul2_rn(make_float2(x.z, x.w), f2(gr[r]));
    }
#pragma unroll
    for (int p = 0; p < 8; ++p)
      part[p] = r == 0 ? __fmul2_rn(T[r][p], f2(kr[r])) : __ffma2_rn(T[r][p], f2(kr[r]), part[p]);
  }
  const float P = column_sum<D>(red, rg, cc, part);
  if ((tid & 1) == 0) {
    const int j = tid >> 1;
    wsh[j] = __fmul_rn(hd.beta, __fsub_rn(S.v()[j], P));
  }
  __syncthreads();
  float2 W[8];
  {
    const float4* wsrc = reinterpret_cast<const float4*>(wsh + 16 * cc);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float4 x = wsrc[p];
      W[2 * p] = make_float2(x.x, x.y);
      W[2 * p + 1] = make_float2(x.z, x.w);
    }
  }
  // delta update, partial S^T q
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      T[r][p] = __ffma2_rn(f2(kr[r]), W[p], T[r][p]);
      part[p] = r == 0 ? __fmul2_rn(T[r][p], f2(qr[r])) : __ffma2_rn(T[r][p], f2(qr[r]), part[p]);
    }
  }
  {
    const float O = column_sum<D>(red, rg, cc, part);
    if ((tid & 1) == 0) {
      const int j = tid >> 1;
      if (O != O) st |= ST_NAN;
      o[j] = O;
    }
  }
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const int i = r * G::NG + rg;
    float4* dst = reinterpret_cast<float4*>(S.rec() + ((size_t)i * D + 16 * cc) * 4);
#pragma unroll
    for (int p = 0; p < 4; ++p)
      dst[p] = make_float4(T[r][2 * p].x, T[r][2 * p].y, T[r][2 * p + 1].x, T[r][2 * p + 1].y);
  }
}

template <int D>
__global__ void __launch_bounds__(Geo<D>::NT, 1) k_decode_step_fp32(const StepArgs a) {
  using G = Geo<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[4];
  __shared__ __align__(16) float wsh[D];
  __shared__ uint32_t st_sh;
  __shared__ int abort_sh;
  float* red = reinterpret_cast<float*>(smem + (size_t)a.nstage * a.stage_bytes);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int cc = lane % G::LPR;
  const int rg = warp * G::RPW + lane / G::LPR;

  const int n_tiles = a.B * a.h_v;
  const int per = (n_tiles + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * per;
  const int t1 = min(n_tiles, t0 + per);
  if (t0 >= t1) return;

  TileScalars pre;  // thread 0: scalars of the next tile to issue
  if (tid == 0) {
    for (int s = 0; s < a.nstage; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    st_sh = 0;
    abort_sh = 0;
    pre = load_scalars<D>(a, t0, t1, false);
    for (int s = 0; s < a.nstage && t0 + s < t1; ++s) {
      const TileScalars cur = pre;
      pre = load_scalars<D>(a, t0 + s + 1, t1, false);
      issue_fp32<D>(a, cur, smem + (size_t)s * a.stage_bytes, &bars[s]);
    }
  }
  __syncthreads();

  uint32_t st = 0;
  for (int n = 0; t0 + n < t1; ++n) {
    const int tile = t0 + n;
    const int sidx = n % a.nstage;
    const uint32_t parity = (uint32_t)(n / a.nstage) & 1u;
    uint8_t* sbase = smem + (size_t)sidx * a.stage_bytes;
    Stage<D> S{sbase, a.rec_cap};
    const bool ok = mbar_wait_bounded(&bars[sidx], parity, 2000000000ull);
    if (!ok) abort_sh = 1;
    __syncthreads();
    if (abort_sh) { st |= ST_TIMEOUT; break; }

    const int b = tile / a.h_v;
    const int h = tile - b * a.h_v;
    float* o = a.o + ((size_t)b * a.h_v + h) * D;
    const TileHdr hd = *S.hdr();
    if (hd.valid) {
      tile_body_fp32<D>(a, S, hd, red, wsh, o, rg, cc, st);
      fence_proxy_async_smem();
    } else {
      if (tid < D) o[tid] = 0.0f;
      st |= ST_SLOT;
    }
    __syncthreads();
    if (tid == 0) {
      if (hd.valid) {
        bulk_s2g(hd.dst, S.rec(), hd.bytes);
        bulk_commit();
        bulk_wait_read_all();  // the stage may be refilled once the store has read it
      }
      if (tile + a.nstage < t1) {
        const TileScalars cur = pre;
        pre = load_scalars<D>(a, tile + a.nstage + 1, t1, false);
        issue_fp32<D>(a, cur, sbase, &bars[sidx]);
      }
    }
  }
  if (st) atomicOr(&st_sh, st);
  __syncthreads();
  if (tid == 0) {
    if (abort_sh) {
      // give in-flight loads a bounded chance to land before the CTA exits
      for (int s = 0; s < a.nstage; ++s) (void)mbar_wait_bounded(&bars[s], 0, 1000000ull);
    }
    bulk_wait_all();
    if (st_sh) atomicOr(a.t.status, st_sh);
  }
}

// ----------------------------------------------------------- packed state
// Scheduling helpers of the persistent packed step (sq_step.cuh). Tiles are
// numbered head-major, m = h B + b, and handed out in chunks of a.chunk
// consecutive tiles from a global counter: a CTA works on one head (one
// width, one code path) for several tiles in a row, and the CTAs stay
// balanced although the widths cost differently.
//
// Control block of the producing thread (shared memory, thread 0 only).
// The scalars of the next tile to issue are fetched with cp.async one
// refill ahead (double-buffered), and the next chunk is claimed one chunk
// ahead, so the producer never waits on global memory inside a tile.
struct Producer {
  int32_t slot[2];
  uint32_t rec_off[2], rec_bytes[2];
  uint32_t kind_word[2];  // the 4-byte word of head_kind holding the head's entry
  float beta[2], g[2];
  int next;  // next tile to issue (head-major index), or -1: no more work
  int end;   // end of the chunk that holds `next`
  int buf;   // scalar buffer holding the scalars of `next`
  int pend;  // stage whose record store is issued and whose refill is pending, or -1
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Thread 0: start fetching the scalars of tile m (head-major) into buffer k.
__device__ __forceinline__ void prefetch_scalars(const StepArgs& a, Producer* pr, int m, int k) {
  if (m < 0) return;
  const int h = m / a.B;
  const int b = m - h * a.B;
  const int bh = b * a.h_v + h;
  if (a.slots)
    cp_async4(&pr->slot[k], a.slots + b);
  else
    pr->slot[k] = b;
  cp_async4(&pr->rec_off[k], a.t.rec_off + h);
  cp_async4(&pr->rec_bytes[k], a.t.rec_bytes + h);
  cp_async4(&pr->kind_word[k], a.t.head_kind + (h & ~3));  // the table is padded to 16 bytes
  cp_async4(&pr->beta[k], a.beta + bh);
  if (a.gate_kind == 0) cp_async4(&pr->g[k], a.g + bh);
  cp_async_commit();
}

// Thread 0: set up the first chunk (the claim of the one after it, `ahead`,
// is in flight when this returns).
__device__ __forceinline__ void producer_start(const StepArgs& a, Producer* pr, int& ahead) {
  const int n_tiles = a.B * a.h_v;
  const int n_chunks = (n_tiles + a.chunk - 1) / a.chunk;
  const int c0 = (int)atomicAdd(a.t.sched, 1u);
  ahead = (int)atomicAdd(a.t.sched, 1u);
  if (c0 < n_chunks) {
    pr->next = c0 * a.chunk;
    pr->end = min(pr->next + a.chunk, n_tiles);
  } else {
    pr->next = -1;
  }
  pr->buf = 0;
  pr->pend = -1;
  prefetch_scalars(a, pr, pr->next, 0);
}

// max(|a|, |b|, |c|), NaN if any input is NaN (one instruction on sm_100).
__device__ __forceinline__ float absmax3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ===================================================== quantize / dequantize
// One CTA per (request, head) tile.
struct QuantArgs {
  uint8_t* pool;
  const float* S;        // quantize: [B, h_v, d, d] input
  float* S_out;          // dequantize: [B, h_v, d, d] output
  const int32_t* slots;
  int32_t B, h_v, n_slots;
  uint64_t slot_bytes;
  Tables t;
};

template <int D>
__global__ void __launch_bounds__(Geo<D>::NT) k_quantize(const QuantArgs a) {
  using G = Geo<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tile = blockIdx.x;
  const int b = tile / a.h_v;
  const int h = tile - b * a.h_v;
  const int slot = a.slots ? a.slots[b] : b;
  const int tid = threadIdx.x;
  if (slot < 0 || slot >= a.n_slots) {
    if (tid == 0) atomicOr(a.t.status, ST_SLOT);
    return;
  }
  const int lane = tid & 31, warp = tid >> 5;
  const int cc = lane % G::LPR;
  const int rg = warp * G::RPW + lane / G::LPR;
  uint8_t* rec = smem;
  const uint32_t rb = a.t.rec_bytes[h];
  uint16_t* row_off = reinterpret_cast<uint16_t*>(smem + rb);
  uint8_t* row_code = reinterpret_cast<uint8_t*>(row_off + D);
  float* phi = reinterpret_cast<float*>(row_code + D);
  for (int i = tid; i < D; i += G::NT) {
    row_off[i] = a.t.row_off[(size_t)h * D + i];
    row_code[i] = a.t.row_code[(size_t)h * D + i];
    phi[i] = a.t.phi[(size_t)h * D + i];
  }
  // zero the record (padding bytes stay zero)
  for (uint32_t x = tid * 16; x < rb; x += G::NT * 16) *reinterpret_cast<uint4*>(rec + x) = make_uint4(0, 0, 0, 0);
  float2 ic[8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
    ic[p] = make_float2(a.t.icol[(size_t)h * D + 16 * cc + 2 * p], a.t.icol[(size_t)h * D + 16 * cc + 2 * p + 1]);
  float2 T[G::RPT][8];
  const float* Sh = a.S + ((size_t)b * a.h_v + h) * D * D;
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const int i = r * G::NG + rg;
    const float4* src = reinterpret_cast<const float4*>(Sh + (size_t)i * D + 16 * cc);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float4 x = src[p];
      T[r][2 * p] = __fmul2_rn(make_float2(x.x, x.y), ic[2 * p]);
      T[r][2 * p + 1] = __fmul2_rn(make_float2(x.z, x.w), ic[2 * p + 1]);
    }
  }
  __syncthreads();
  uint32_t st = requant_rows<D, 0>(rec, row_off, row_code, phi, rg, cc, false, T);
  __syncthreads();
  uint8_t* dst = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[h];
  for (uint32_t x = tid * 16; x < rb; x += G::NT * 16) *reinterpret_cast<uint4*>(dst + x) = *reinterpret_cast<uint4*>(rec + x);
  if (st) atomicOr(a.t.status, st);
}

template <int D>
__global__ void __launch_bounds__(Geo<D>::NT) k_dequantize(const QuantArgs a) {
  using G = Geo<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tile = blockIdx.x;
  const int b = tile / a.h_v;
  const int h = tile - b * a.h_v;
  const int slot = a.slots ? a.slots[b] : b;
  const int tid = threadIdx.x;
  float* Sh = a.S_out + ((size_t)b * a.h_v + h) * D * D;
  if (slot < 0 || slot >= a.n_slots) {
    for (int x = tid; x < D * D / 4; x += G::NT) reinterpret_cast<float4*>(Sh)[x] = make_float4(0, 0, 0, 0);
    if (tid == 0) atomicOr(a.t.status, ST_SLOT);
    return;
  }
  const int lane = tid & 31, warp = tid >> 5;
  const int cc = lane % G::LPR;
  const int rg = warp * G::RPW + lane / G::LPR;
  uint8_t* rec = smem;
  const uint32_t rb = a.t.rec_bytes[h];
  const uint8_t* src = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[h];
  for (uint32_t x = tid * 16; x < rb; x += G::NT * 16) *reinterpret_cast<uint4*>(rec + x) = *reinterpret_cast<const uint4*>(src + x);
  __syncthreads();
  float2 c[8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
    c[p] = make_float2(a.t.col[(size_t)h * D + 16 * cc + 2 * p], a.t.col[(size_t)h * D + 16 * cc + 2 * p + 1]);
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const int i = r * G::NG + rg;
    const uint8_t code = a.t.row_code[(size_t)h * D + i];
    const uint8_t* row = rec + a.t.row_off[(size_t)h * D + i];
    float2 T[8];
    const float mul = code == ROW_PIVOT ? 1.0f : __half2float(reinterpret_cast<const __half*>(rec)[i]);
    load_row(row, code, cc, mul, T);
    float4* dst = reinterpret_cast<float4*>(Sh + (size_t)i * D + 16 * cc);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float2 s0 = __fmul2_rn(T[2 * p], c[2 * p]);
      float2 s1 = __fmul2_rn(T[2 * p + 1], c[2 * p + 1]);
      dst[p] = make_float4(s0.x, s0.y, s1.x, s1.y);
    }
  }
}

// FP32 pools: plain tile copies between S [B, h_v, d, d] and pool slots.
template <int D>
__global__ void k_copy_fp32(float* pool, const float* S_in, float* S_out, const int32_t* slots, int h_v, int n_slots,
                            uint32_t* status) {
  const int tile = blockIdx.x;
  const int b = tile / h_v;
  const int h = tile - b * h_v;
  const int slot = slots ? slots[b] : b;
  const size_t n4 = (size_t)D * D / 4;
  if (slot < 0 || slot >= n_slots) {
    if (S_out)
      for (size_t x = threadIdx.x; x < n4; x += blockDim.x)
        reinterpret_cast<float4*>(S_out + ((size_t)b * h_v + h) * D * D)[x] = make_float4(0, 0, 0, 0);
    if (threadIdx.x == 0) atomicOr(status, ST_SLOT);
    return;
  }
  float4* P = reinterpret_cast<float4*>(pool + ((size_t)slot * h_v + h) * D * D);
  if (S_in) {
    const float4* src = reinterpret_cast<const float4*>(S_in + ((size_t)b * h_v + h) * D * D);
    for (size_t x = threadIdx.x; x < n4; x += blockDim.x) P[x] = src[x];
  } else {
    float4* dst = reinterpret_cast<float4*>(S_out + ((size_t)b * h_v + h) * D * D);
    for (size_t x = threadIdx.x; x < n4; x += blockDim.x) dst[x] = P[x];
  }
}

}  // namespace sqk
