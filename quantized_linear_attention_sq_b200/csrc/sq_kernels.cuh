// sq_kernels.cuh -- sm_100a kernels of the quantized-state decode step.
//
// One CTA owns one (request, value head) state tile at a time. CTAs are
// persistent: each walks a contiguous run of tiles, and its records (plus
// the tile's small vectors and the head's calibration rows) arrive in shared
// memory through 1-D TMA bulk copies (cp.async.bulk, no multicast) completed
// on an mbarrier, NSTAGE tiles ahead of the one being computed. The updated
// record is written back in place from shared memory with a bulk store. The
// state therefore crosses HBM exactly once in each direction per step
// ("STEPQuant: estados recurrentes a 6 bit" (gpt-diffusion), section "Las
// dos ideas": fused kernels that move the packed state, not FP32).
//
// Thread map for a d x d tile: a thread owns 16 consecutive value columns of
// RPT key rows (d = 128: 256 threads, 4 rows each; 8 lanes cover one row, so
// a row's 16-column chunk is 2*b bytes = b/2 whole 32-bit words for every
// width b). Column sums (S^T k, S^T q) go through shared memory; row maxima
// use warp shuffles over the 8 lanes of a row.
//
// Arithmetic follows a fixed elementwise recipe so that codes are
// reproducible: a_i = r_i g_i; T = q a_i; P_j = sum_i T_ij k_i;
// u_j = beta (v_j - c_j P_j); w_j = u_j / c_j (as u_j * fl(1/c_j));
// T' = fma(k_i, w_j, T); o_j = c_j sum_i T'_ij q_i; m_i = max_j |T'_ij|;
// r'_i = fp16 round-up of (phi_i m_i) / qmax; q' = RNE(clamp(T' * fl(1/r'))).
// Only the two column sums depend on summation order.
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
  const float* col;           // [h_v*d] c_j
  const float* icol;          // [h_v*d] fl(1 / c_j)
  const float* phi;           // [h_v*d] phi_i
  const uint8_t* head_kind;   // [h_v] width shared by all rows of the head (ROW_PIVOT: all pivot), 0: mixed
  uint32_t* status;           // device status word
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
  uint32_t rec_cap;     // bytes reserved for a record in a stage (multiple of 128)
  uint32_t stage_bytes; // rec_cap + aux bytes, multiple of 128
  uint64_t slot_bytes;
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
  static constexpr int AUX = 31 * D + 32;     // aux bytes per stage (see stage layout)
  static_assert(RPT >= 1 && RPT * NG == D, "bad geometry");
};

// Stage layout: [record: rec_cap][k f32 D][q f32 D][v f32 D][g f32 D]
//               [c f32 D][ic f32 D][phi f32 D][row_off u16 D][row_code u8 D]
//               [TileHdr 32 B]
template <int D>
struct Stage {
  uint8_t* base;
  uint32_t rec_cap;
  __device__ uint8_t* rec() const { return base; }
  __device__ float* k() const { return reinterpret_cast<float*>(base + rec_cap); }
  __device__ float* q() const { return k() + D; }
  __device__ float* v() const { return k() + 2 * D; }
  __device__ float* g() const { return k() + 3 * D; }
  __device__ float* c() const { return k() + 4 * D; }
  __device__ float* ic() const { return k() + 5 * D; }
  __device__ float* phi() const { return k() + 6 * D; }
  __device__ uint16_t* row_off() const { return reinterpret_cast<uint16_t*>(k() + 7 * D); }
  __device__ uint8_t* row_code() const { return reinterpret_cast<uint8_t*>(row_off() + D); }
  __device__ struct TileHdr* hdr() const { return reinterpret_cast<struct TileHdr*>(row_code() + D); }
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
  uint32_t pad;
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

// Exponent E of the fp64 view of a field: the field sits at bits
// [20-E, 20-E+B) of the word 0x3FF00000, so that, read as the high word of a
// double (low word 0), the word is 1 + field * 2^-E exactly and, read as a
// float, 1.875 + field * 2^-(E+3). 8-bit fields go to a byte boundary
// (E = 12) so one byte permute places them; the others use E = B.
template <int B>
struct FieldPos {
  static constexpr int E = B == 8 ? 12 : B;
  static constexpr int POS = 20 - E;
};

// Field j of a 16-code chunk held in b/2 words, in place as described above.
template <int B>
__device__ __forceinline__ uint32_t field_hi(const uint32_t* w, int j) {
  constexpr int POS = FieldPos<B>::POS;
  if constexpr (B == 8) {
    return __byte_perm(w[j >> 2], 0x3FF00000u, 0x7604u | ((uint32_t)(j & 3) << 4));
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
    return 0x3FF00000u | (x & MASK);
  }
}

// Pass-A unpack of one quantized 16-code chunk: the codes q as floats (exact)
// and the high words of the doubles 1 + field * 2^-E that feed the fp64
// column sum (with the per-row factor 2^E a k, minus (1 + 2^(B-1-E)) 2^E a k
// per row, they give q a k up to fp64 rounding).
template <int B>
__device__ __forceinline__ void unpack_q_hi(const uint8_t* row, int cc, float2 (&V)[8], uint32_t (&xh)[16]) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 2 * B * cc);
  uint32_t w[B / 2];
#pragma unroll
  for (int i = 0; i < B / 2; ++i) w[i] = src[i];
  constexpr int E = FieldPos<B>::E;
  const float S = (float)(1 << (E + 3));
  const float C = 1.875f * S + (float)(1 << (B - 1));
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint32_t h0 = field_hi<B>(w, 2 * p), h1 = field_hi<B>(w, 2 * p + 1);
    xh[2 * p] = h0;
    xh[2 * p + 1] = h1;
    V[p] = __ffma2_rn(make_float2(__uint_as_float(h0), __uint_as_float(h1)), make_float2(S, S),
                      make_float2(-C, -C));
  }
}

// Pass-A unpack of one fp16 pivot chunk: the values as floats and the high
// words of the same values as doubles (an fp16 value has a zero low word).
__device__ __forceinline__ void unpack_pivot_hi(const uint8_t* row, int cc, float2 (&V)[8], uint32_t (&xh)[16]) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 32 * cc);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    __half2 h2 = *reinterpret_cast<const __half2*>(src + p);
    float2 x = __half22float2(h2);
    V[p] = x;
    xh[2 * p] = (uint32_t)__double2hiint((double)x.x);
    xh[2 * p + 1] = (uint32_t)__double2hiint((double)x.y);
  }
}

__device__ __forceinline__ void unpack_hi(const uint8_t* row, uint8_t code, int cc, float2 (&V)[8],
                                          uint32_t (&xh)[16]) {
  switch (code) {
    case 8: unpack_q_hi<8>(row, cc, V, xh); break;
    case 6: unpack_q_hi<6>(row, cc, V, xh); break;
    case 4: unpack_q_hi<4>(row, cc, V, xh); break;
    case 2: unpack_q_hi<2>(row, cc, V, xh); break;
    default: unpack_pivot_hi(row, cc, V, xh); break;
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

// Requantize one row chunk of T' with inverse scale `ir` and write it back.
// fma(T', ir, 2^23 + 2^(b-1)) rounds the exact product T' * ir to the
// nearest integer (ties to even) in the window [2^23, 2^24) where floats
// are integers; outside that window the value lies beyond the clamp bounds
// whichever way it rounds, so clamping afterwards gives exactly the clamped
// nearest integer. The result's low b bits are then the stored field.
template <int B>
__device__ __forceinline__ void store_row_q(uint8_t* row, int cc, float ir, const float2 (&t)[8]) {
  const float qm = (float)((1 << (B - 1)) - 1);
  const float magic = 8388608.0f + (float)(1 << (B - 1));
  const float lo = magic - qm, hi = magic + qm;
  uint32_t fb[16];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float2 n = __ffma2_rn(t[p], f2(ir), f2(magic));
    n.x = fminf(fmaxf(n.x, lo), hi);
    n.y = fminf(fmaxf(n.y, lo), hi);
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

// fp16 pivot row: RNE with saturation at +-65504; NaN stores 0.
__device__ __forceinline__ uint32_t store_row_pivot(uint8_t* row, int cc, const float2 (&t)[8]) {
  uint32_t st = 0;
  uint32_t* dst = reinterpret_cast<uint32_t*>(row + 32 * cc);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float x0 = t[p].x, x1 = t[p].y;
    if (x0 != x0) { x0 = 0.0f; st |= ST_NAN; }
    if (x1 != x1) { x1 = 0.0f; st |= ST_NAN; }
    if (fabsf(x0) > 65504.0f) { x0 = copysignf(65504.0f, x0); st |= ST_SAT; }
    if (fabsf(x1) > 65504.0f) { x1 = copysignf(65504.0f, x1); st |= ST_SAT; }
    __half2 h = __floats2half2_rn(x0, x1);
    dst[p] = *reinterpret_cast<uint32_t*>(&h);
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
  float ir_m = 0.0f;
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
      rbits = __half_as_ushort(rh);
    }
  }
  if (cc < G::RPT) reinterpret_cast<uint16_t*>(rec)[im] = rbits;
  const int lane = threadIdx.x & 31;
  const int base = lane - cc;
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
    const float ir = __shfl_sync(0xffffffffu, ir_m, base + r);
    const int i = r * G::NG + rg;
    const int code = KC ? KC : row_code[i];
    uint8_t* row = rec + row_offset<D, KC>(row_off, i);
    if (code == ROW_PIVOT) {
      st |= store_row_pivot(row, cc, T[r]);
    } else if (m[r] != m[r]) {  // a NaN in the row: scale 0, all codes 0
      store_row_zero(row, code, cc);
    } else {
      switch (code) {
        case 8: store_row_q<8>(row, cc, ir, T[r]); break;
        case 6: store_row_q<6>(row, cc, ir, T[r]); break;
        case 4: store_row_q<4>(row, cc, ir, T[r]); break;
        default: store_row_q<2>(row, cc, ir, T[r]); break;
      }
    }
  }
  return st;
}

// Column sums. Every thread deposits its 16 partials for its row group;
// a thread's chunks are stored rotated by its column block (XOR swizzle) so
// the eight lanes of a row write eight different bank groups. Then two
// adjacent threads own one column (thread 2j and 2j+1 each add half of the
// row groups) and combine with one shuffle. Returns the column total in
// every thread of the pair; column = threadIdx.x >> 1. The caller syncs
// before reusing `red`.
template <int D>
__device__ __forceinline__ float column_sum(float* red, int rg, int cc, const float2 (&part)[8]) {
  using G = Geo<D>;
  static_assert(G::NT == 2 * D, "two threads per column");
  const int sw = (cc >> 1) & 3;
#pragma unroll
  for (int p = 0; p < 4; ++p)
    *reinterpret_cast<float4*>(red + rg * D + 16 * cc + 4 * (p ^ sw)) =
        make_float4(part[2 * p].x, part[2 * p].y, part[2 * p + 1].x, part[2 * p + 1].y);
  __syncthreads();
  const int j = threadIdx.x >> 1;
  const int hh = threadIdx.x & 1;
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 4 * ((e >> 2) ^ ((cj >> 1) & 3)) + (e & 3);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int g = 0; g < G::NG / 2; g += 2) {
    a0 = __fadd_rn(a0, red[(hh * (G::NG / 2) + g) * D + off]);
    a1 = __fadd_rn(a1, red[(hh * (G::NG / 2) + g + 1) * D + off]);
  }
  const float a = __fadd_rn(a0, a1);
  return __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 1));
}

// fp64 deposit of the 16 pass-A partials (same swizzle idea, 16-byte chunks
// of two doubles rotated by cc).
template <int D>
__device__ __forceinline__ void deposit_f64(double* red, int rg, int cc, int half, const double (&acc)[8],
                                            double off) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int chunk = 4 * half + p;
    *reinterpret_cast<double2*>(red + rg * D + 16 * cc + 2 * (chunk ^ (cc & 7))) =
        make_double2(acc[2 * p] - off, acc[2 * p + 1] - off);
  }
}

// Column total of the fp64 partials, rounded once to fp32 (two threads per
// column as in column_sum; column = threadIdx.x >> 1). Syncs first.
template <int D>
__device__ __forceinline__ float column_total_f64(const double* red) {
  using G = Geo<D>;
  __syncthreads();
  const int j = threadIdx.x >> 1;
  const int hh = threadIdx.x & 1;
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 2 * ((e >> 1) ^ (cj & 7)) + (e & 1);
  double a0 = 0.0, a1 = 0.0;
#pragma unroll
  for (int g = 0; g < G::NG / 2; g += 2) {
    a0 += red[(hh * (G::NG / 2) + g) * D + off];
    a1 += red[(hh * (G::NG / 2) + g + 1) * D + off];
  }
  const double a = a0 + a1;
  return __double2float_rn(a + __shfl_xor_sync(0xffffffffu, a, 1));
}

// ================================================================ step kernel
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

template <int D>
__device__ __forceinline__ void issue_tile(const StepArgs& a, const TileScalars& x, uint8_t* stage_base,
                                           uint64_t* bar, bool packed) {
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
  uint8_t* rec_src = packed ? a.pool + (uint64_t)x.slot * a.slot_bytes + x.rec_off
                            : a.pool + ((uint64_t)x.slot * a.h_v + h) * (uint64_t)(4u * D * D);
  hd->dst = rec_src;
  hd->bytes = x.rec_bytes;
  hd->valid = 1;
  hd->beta = x.beta;
  hd->g = x.g;
  hd->kind = x.kind;
  uint32_t tx = x.rec_bytes + 3 * vec + (kda ? vec : 0u);
  if (packed) tx += 3 * vec + 2u * D + (uint32_t)D;
  mbar_arrive_expect_tx(bar, tx);  // release: the header stores above become visible with the phase
  bulk_g2s(s.rec(), rec_src, x.rec_bytes, bar);
  bulk_g2s(s.k(), a.k + ((size_t)b * a.h_k + hk) * D, vec, bar);
  bulk_g2s(s.q(), a.q + ((size_t)b * a.h_k + hk) * D, vec, bar);
  bulk_g2s(s.v(), a.v + ((size_t)b * a.h_v + h) * D, vec, bar);
  if (kda) bulk_g2s(s.g(), a.g + ((size_t)b * a.h_v + h) * D, vec, bar);
  if (packed) {
    bulk_g2s(s.c(), a.t.col + (size_t)h * D, vec, bar);
    bulk_g2s(s.ic(), a.t.icol + (size_t)h * D, vec, bar);
    bulk_g2s(s.phi(), a.t.phi + (size_t)h * D, vec, bar);
    bulk_g2s(s.row_off(), a.t.row_off + (size_t)h * D, 2u * D, bar);
    bulk_g2s(s.row_code(), a.t.row_code + (size_t)h * D, (uint32_t)D, bar);
  }
}

// The compute of one tile, from the stage in shared memory to the updated
// record written back into the stage and o written to global memory. KC is
// the width shared by every row of the head (ROW_PIVOT for an all-pivot
// head), known at compile time, or 0 for heads whose rows differ (KDA):
// with KC != 0 every per-row width switch folds away.
template <int D, bool PACKED, int KC>
__device__ __forceinline__ void tile_body(const StepArgs& a, const Stage<D>& S, const TileHdr& hd, float* red,
                                          float* wsh, int* nf_sh, float* o, int rg, int cc, uint32_t& st) {
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

  // ---- pass A: values, gate, column sum S^T k
  // packed: T holds the stored values V (codes or fp16) and mr the per-row
  // multiplier M (a_i = r_i g_i, or g_i for a pivot row); the column sum
  // is accumulated in fp64 from the exact per-row factors (see unpack_hi),
  // in two halves of 8 columns to keep the accumulators few.
  // fp32: T holds the gated state g_i S_ij and the column sum is fp32.
  float2 T[G::RPT][8];
  float mr[G::RPT];
  float2 part[8];
  float P;
  if (PACKED) {
    double kap[G::RPT];
    double off = 0.0;
    bool bad = false;
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      const int i = r * G::NG + rg;
      const int code = KC ? KC : S.row_code()[i];
      if (code == ROW_PIVOT) {
        mr[r] = gr[r];
        kap[r] = (double)gr[r] * (double)kr[r];
      } else {
        const float R = __half2float(reinterpret_cast<const __half*>(S.rec())[i]);
        mr[r] = __fmul_rn(R, gr[r]);
        const int E = code == 8 ? 12 : code;  // FieldPos<code>::E
        kap[r] = (double)mr[r] * (double)kr[r] * (double)(1 << E);
        off = off + (1.0 + (double)(1 << (code - 1)) / (double)(1 << E)) * kap[r];
      }
      bad |= !isfinite(mr[r]) || !isfinite(kr[r]);
    }
    double* red64 = reinterpret_cast<double*>(red);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      double acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.0;
#pragma unroll
      for (int r = 0; r < G::RPT; ++r) {
        const int i = r * G::NG + rg;
        const int code = KC ? KC : S.row_code()[i];
        const uint8_t* row = S.rec() + row_offset<D, KC>(S.row_off(), i);
        // unpack through temporaries: writing T[r] from inside the width
        // switch would push the whole tile into local memory
        float2 vt[8];
        uint32_t xh[16];
        unpack_hi(row, code, cc, vt, xh);
#pragma unroll
        for (int p = 0; p < 4; ++p) T[r][4 * half + p] = vt[4 * half + p];
        if (code == ROW_PIVOT) {
#pragma unroll
          for (int p = 0; p < 4; ++p) bad |= !isfinite(vt[4 * half + p].x) || !isfinite(vt[4 * half + p].y);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = fma(__hiloint2double((int)xh[8 * half + j], 0), kap[r], acc[j]);
      }
      deposit_f64<D>(red64, rg, cc, half, acc, off);
    }
    if (bad) *nf_sh = 1;
    P = column_total_f64<D>(red64);
  } else {
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
    P = column_sum<D>(red, rg, cc, part);
  }
  if ((tid & 1) == 0) {
    const int j = tid >> 1;
    float wj;
    if (PACKED) {
      const float p = __fmul_rn(S.c()[j], P);
      const float u = __fmul_rn(hd.beta, __fsub_rn(S.v()[j], p));
      wj = __fmul_rn(u, S.ic()[j]);
      if (!isfinite(wj)) *nf_sh = 1;
    } else {
      wj = __fmul_rn(hd.beta, __fsub_rn(S.v()[j], P));
    }
    wsh[j] = wj;
  }
  __syncthreads();
  const bool finite = *nf_sh == 0;
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
  // ---- pass B: gate + delta update (one rounding), partial S^T q
#pragma unroll
  for (int r = 0; r < G::RPT; ++r) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if (PACKED) {
        const float2 kw = __fmul2_rn(f2(kr[r]), W[p]);
        T[r][p] = __ffma2_rn(T[r][p], f2(mr[r]), kw);
      } else {
        T[r][p] = __ffma2_rn(f2(kr[r]), W[p], T[r][p]);
      }
      part[p] = r == 0 ? __fmul2_rn(T[r][p], f2(qr[r])) : __ffma2_rn(T[r][p], f2(qr[r]), part[p]);
    }
  }
  {
    const float O = column_sum<D>(red, rg, cc, part);
    if ((tid & 1) == 0) {
      const int j = tid >> 1;
      const float oj = PACKED ? __fmul_rn(S.c()[j], O) : O;
      if (oj != oj) st |= ST_NAN;
      o[j] = oj;
    }
  }
  // ---- requantize (or store fp32) into the stage record, in place
  if (PACKED) {
    st |= requant_rows<D, KC>(S.rec(), S.row_off(), S.row_code(), S.phi(), rg, cc, finite, T);
  } else {
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      const int i = r * G::NG + rg;
      float4* dst = reinterpret_cast<float4*>(S.rec() + ((size_t)i * D + 16 * cc) * 4);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        dst[p] = make_float4(T[r][2 * p].x, T[r][2 * p].y, T[r][2 * p + 1].x, T[r][2 * p + 1].y);
    }
  }
}

// PACKED = true: quantized pool; false: fp32 S pool (unquantized baseline).
template <int D, bool PACKED>
__global__ void __launch_bounds__(Geo<D>::NT, PACKED ? 2 : 1) k_decode_step(const StepArgs a) {
  using G = Geo<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[4];
  __shared__ __align__(16) float wsh[D];
  __shared__ uint32_t st_sh;
  __shared__ int abort_sh;
  __shared__ int nf_sh;  // the current tile saw a non-finite input
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
    nf_sh = 0;
    pre = load_scalars<D>(a, t0, t1, PACKED);
    for (int s = 0; s < a.nstage && t0 + s < t1; ++s) {
      const TileScalars cur = pre;
      pre = load_scalars<D>(a, t0 + s + 1, t1, PACKED);
      issue_tile<D>(a, cur, smem + (size_t)s * a.stage_bytes, &bars[s], PACKED);
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
    if (!hd.valid) {
      if (tid < D) o[tid] = 0.0f;  // (nf_sh stays 0: nothing was computed)
      st |= ST_SLOT;
      // nothing was loaded into this stage; refill it if there is work left
      __syncthreads();
      if (tid == 0 && tile + a.nstage < t1) {
        const TileScalars cur = pre;
        pre = load_scalars<D>(a, tile + a.nstage + 1, t1, PACKED);
        issue_tile<D>(a, cur, sbase, &bars[sidx], PACKED);
      }
      continue;
    }

    switch (PACKED ? hd.kind : 0) {
      case 8: tile_body<D, PACKED, (PACKED ? 8 : 0)>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st); break;
      case 6: tile_body<D, PACKED, (PACKED ? 6 : 0)>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st); break;
      case 4: tile_body<D, PACKED, (PACKED ? 4 : 0)>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st); break;
      case 2: tile_body<D, PACKED, (PACKED ? 2 : 0)>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st); break;
      case ROW_PIVOT:
        tile_body<D, PACKED, (PACKED ? ROW_PIVOT : 0)>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st);
        break;
      default: tile_body<D, PACKED, 0>(a, S, hd, red, wsh, &nf_sh, o, rg, cc, st); break;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      nf_sh = 0;  // every read of this tile's flag happened before the barrier above
      bulk_s2g(hd.dst, S.rec(), hd.bytes);
      bulk_commit();
      bulk_wait_read_all();  // the stage may be refilled once the store has read it
      if (tile + a.nstage < t1) {
        const TileScalars cur = pre;
        pre = load_scalars<D>(a, tile + a.nstage + 1, t1, PACKED);
        issue_tile<D>(a, cur, sbase, &bars[sidx], PACKED);
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
