// sq_step.cuh -- the fused decode step on a packed state pool (sm_100a).
//
// For every (request, value head) tile: read the packed record once, form
// S^T k from the stored codes, apply gate and delta update, emit o, refresh
// the row scales and requantize and repack the tile in place, writing it
// once ("STEPQuant: estados recurrentes a 6 bit" (gpt-diffusion), section
// "Las dos ideas": fused kernels that move the packed state, not FP32).
//
// Work distribution. Persistent CTAs of D threads (D = 128: 4 warps, 4 CTAs
// per SM) take tiles one at a time from a global counter, tiles numbered
// head major so that a CTA stays on one width for long runs. Thread 0 issues
// 1-D TMA bulk copies (cp.async.bulk, no multicast) of the record and the
// tile's vectors into one of two shared-memory stages, completed on an
// mbarrier; the updated record goes back from the stage with a bulk store.
//
// Thread map: a thread owns 16 consecutive value columns of RPT = D/16 key
// rows (row slots r * 16 + rg, r < RPT; 16 row groups rg); the RPT lanes of
// a row group cover one row. The tile is not kept in registers:
//   pass A  codes -> S^T k partials in fp64, deposited per row group;
//   B1      column totals (one thread per column), the rounding of each
//           total to fp32 certified against an error bound, w;
//   B2      pass B: codes unpacked again, T' = fma(V, M, k w), o partials,
//           requantization QS rows at a time, new codes written in place;
//   B3      o totals; thread 0 stores the record.
//
// S^T k is defined as the exact value of sum_i V_ij M_i k_i rounded once to
// fp32 (ties to even). Pass A sums the products in fp64 (each thread over
// its RPT rows, then 16 partials per column); the tile's rigorous bound eps
// on |fp64 total - exact value| (below) decides: when every value within
// eps of the total rounds to the same fp32 number, that number is the
// rounding of the exact value; otherwise the warp sums the column again in
// double-double arithmetic (column_warp, certified the same way) and, on an
// exact tie, with a fixed-point accumulator (exact_column). Either way P_j
// is the exact value rounded once, independent of summation order.
#pragma once

#include "sq_kernels.cuh"

namespace sqk {

// Stages of the packed step (the kernel's mbarrier array has this many
// entries; the host plans exactly this many).
constexpr int kPackedStages = 2;

template <int D>
struct PGeo {
  static constexpr int LPR = D / 16;    // lanes per key row (16 columns each)
  static constexpr int RPW = 32 / LPR;  // rows a warp covers per pass
  static constexpr int NG = 16;         // row groups
  static constexpr int NW = NG / RPW;   // warps per CTA
  static constexpr int NT = 32 * NW;    // threads per CTA (= D: one per column)
  static constexpr int RPT = D / NG;    // rows per thread (= LPR)
  static constexpr int QS = RPT < 4 ? RPT : 4;  // rows requantized together
  // stage vectors: [k f32 D][q f32 D][g f32 D][phi f32 D][row_off u16 D]
  //                [row_code u8 D][row_perm u8 D][TileHdr 32 B], then the record
  //                (rec_cap bytes) and 2 D bytes of slack
  static constexpr uint32_t AUX = (uint32_t)((20 * D + 32 + 127) / 128 * 128);
  static_assert(NT == D && RPT == LPR && RPT % QS == 0, "geometry");
};

template <int D>
struct PStage {
  uint8_t* base;
  __device__ float* k() const { return reinterpret_cast<float*>(base); }
  __device__ float* q() const { return k() + D; }
  __device__ float* g() const { return k() + 2 * D; }
  __device__ float* phi() const { return k() + 3 * D; }
  __device__ uint16_t* row_off() const { return reinterpret_cast<uint16_t*>(k() + 4 * D); }
  __device__ uint8_t* row_code() const { return reinterpret_cast<uint8_t*>(row_off() + D); }
  __device__ uint8_t* row_perm() const { return row_code() + D; }
  __device__ TileHdr* hdr() const { return reinterpret_cast<TileHdr*>(row_perm() + D); }
  __device__ uint8_t* rec() const { return base + PGeo<D>::AUX; }
};

// ------------------------------------------------------------ exact sum
// Exact sum_i V_ij M_i k_i of one column, rounded once to fp32 (ties to
// even, +0 for an exact zero), for finite inputs. Every term is an integer
// times a power of two: V is an integer code (|V| < 2^7) or an fp16 value
// (11-bit significand), M and k are fp32 (24-bit significands), so a term is
// a 59-bit integer times 2^e with e >= -24 - 149 - 149 = -322 and
// e + 59 <= 5 + 104 + 104 + 59 = 272. The accumulator holds XL limbs of 32
// bits (bit 0 = 2^-352) in int64s, so 128 terms add without carries
// leaving a limb; it is normalised once at the end. Used only for columns
// whose sum the double-double pass (column_warp) cannot round with
// certainty, i.e. in practice exact ties.
namespace xs {
constexpr int XL = 20;
constexpr int LSB = -352;

__device__ __forceinline__ void split32(float x, uint64_t& m, int& e) {
  const uint32_t b = __float_as_uint(x);
  const uint32_t ex = (b >> 23) & 0xFFu;
  m = b & 0x7FFFFFu;
  if (ex) {
    m |= 0x800000u;
    e = (int)ex - 150;
  } else {
    e = -149;
  }
}
__device__ __forceinline__ void split16(uint16_t h, uint64_t& m, int& e) {
  const uint32_t ex = (h >> 10) & 0x1Fu;
  m = h & 0x3FFu;
  if (ex) {
    m |= 0x400u;
    e = (int)ex - 25;
  } else {
    e = -24;
  }
}
}  // namespace xs

// V of row i, column j: the code (quantized row of width `code`) or the
// fp16 bits (pivot row), from the row's bytes.
__device__ __forceinline__ void stored_value(const uint8_t* row, int code, int j, int& qv, uint16_t& hv) {
  if (code == ROW_PIVOT) {
    hv = reinterpret_cast<const uint16_t*>(row)[j];
    qv = 0;
    return;
  }
  const int bit = code * j;
  const uint32_t lo = row[bit >> 3];
  const uint32_t hi = ((bit & 7) + code > 8) ? row[(bit >> 3) + 1] : 0u;
  const uint32_t field = ((lo | (hi << 8)) >> (bit & 7)) & ((1u << code) - 1u);
  qv = (int)field - (1 << (code - 1));
  hv = 0;
}

template <int D>
__device__ __noinline__ float exact_column(const uint8_t* rec, const uint16_t* row_off, const uint8_t* row_code,
                                           int kc, uint32_t rec_cap, const float* M, const float* k, int j) {
  int64_t acc[xs::XL];
#pragma unroll
  for (int l = 0; l < xs::XL; ++l) acc[l] = 0;
  for (int i = 0; i < D; ++i) {
    const int code = kc ? kc : row_code[i];
    const uint32_t off = kc ? (kc == ROW_PIVOT ? 2u * D + (uint32_t)i * 2u * D : 2u * D + (uint32_t)i * (D * kc / 8))
                            : min((uint32_t)row_off[i], rec_cap);
    int qv;
    uint16_t hv;
    stored_value(rec + off, code, j, qv, hv);
    uint64_t mv, mm, mk;
    int ev, em, ek;
    bool neg;
    if (code == ROW_PIVOT) {
      xs::split16(hv, mv, ev);
      neg = (hv >> 15) != 0;
    } else {
      mv = (uint64_t)(qv < 0 ? -qv : qv);
      ev = 0;
      neg = qv < 0;
    }
    xs::split32(M[i], mm, em);
    xs::split32(k[i], mk, ek);
    neg ^= (__float_as_uint(M[i]) >> 31) != 0;
    neg ^= (__float_as_uint(k[i]) >> 31) != 0;
    const uint64_t mag = mv * (mm * mk);  // < 2^11 * 2^48
    if (mag == 0) continue;
    const int pos = ev + em + ek - xs::LSB;  // >= 30
    const int li = pos >> 5, sh = pos & 31;
    const uint64_t lo = mag << sh;
    const uint64_t hi = sh ? (mag >> (64 - sh)) : 0ull;
    const int64_t p0 = (int64_t)(lo & 0xFFFFFFFFull), p1 = (int64_t)(lo >> 32), p2 = (int64_t)hi;
    if (neg) {
      acc[li] -= p0;
      acc[li + 1] -= p1;
      acc[li + 2] -= p2;
    } else {
      acc[li] += p0;
      acc[li + 1] += p1;
      acc[li + 2] += p2;
    }
  }
  // normalise: limbs 0 .. XL-2 in [0, 2^32), the sign in the top limb
  for (int l = 0; l + 1 < xs::XL; ++l) {
    const int64_t c = acc[l] >> 32;
    acc[l] -= c * 4294967296ll;
    acc[l + 1] += c;
  }
  const bool neg = acc[xs::XL - 1] < 0;
  if (neg) {
    for (int l = 0; l < xs::XL; ++l) acc[l] = -acc[l];
    for (int l = 0; l + 1 < xs::XL; ++l) {
      const int64_t c = acc[l] >> 32;
      acc[l] -= c * 4294967296ll;
      acc[l + 1] += c;
    }
  }
  int top = -1;
  for (int l = xs::XL - 1; l >= 0 && top < 0; --l)
    if (acc[l]) top = 32 * l + 63 - __clzll((unsigned long long)acc[l]);
  if (top < 0) return 0.0f;
  int qexp = top + xs::LSB - 23;
  if (qexp < -149) qexp = -149;
  const int q0 = qexp - xs::LSB;  // bit index of the last place kept
  auto bit = [&](int n) -> uint32_t { return n < 0 ? 0u : (uint32_t)((acc[n >> 5] >> (n & 31)) & 1); };
  uint32_t n = 0;
  for (int b = top; b >= q0; --b) n = (n << 1) | bit(b);
  const uint32_t half = bit(q0 - 1);
  uint32_t sticky = 0;
  for (int b = q0 - 2; b >= 0 && !sticky; --b) sticky = bit(b);
  if (half && (sticky || (n & 1u))) ++n;
  float r;
  if (qexp + (n >= (1u << 24) ? 24 : 23) > 127) {
    r = __int_as_float(0x7F800000);
  } else {
    r = scalbnf((float)n, qexp);  // n < 2^25 is exact in fp32 when n <= 2^24 (n = 2^24 only after rounding up)
  }
  return neg ? -r : r;
}

// The same column sum, computed by the 32 lanes of a warp together and
// exact to about 2^-88 of sum |V M k|: every product V (M k) is split
// exactly into a double p and its error e (fma), the 2D doubles are summed
// with error-free additions (TwoSum) into a pair s + c, whose remaining
// error comes only from the additions into c. A bound on that error
// certifies the rounding as before; only a value within that bound of a
// rounding boundary (in practice: an exact tie) goes on to exact_column.
// Every lane must call it with the same j; every lane returns P_j.
__device__ __forceinline__ void two_sum(double a, double b, double& s, double& e) {
  s = a + b;
  const double bb = s - a;
  e = (a - (s - bb)) + (b - bb);
}

template <int D>
__device__ __noinline__ float column_warp(const uint8_t* rec, const uint16_t* row_off, const uint8_t* row_code, int kc,
                                          uint32_t rec_cap, const float* M, const float* k, int j) {
  const int lane = threadIdx.x & 31;
  double s = 0.0, c = 0.0, mag = 0.0;
  for (int i = lane; i < D; i += 32) {
    const int code = kc ? kc : row_code[i];
    const uint32_t off = kc ? (kc == ROW_PIVOT ? 2u * D + (uint32_t)i * 2u * D : 2u * D + (uint32_t)i * (D * kc / 8))
                            : min((uint32_t)row_off[i], rec_cap);
    int qv;
    uint16_t hv;
    stored_value(rec + off, code, j, qv, hv);
    const double V = code == ROW_PIVOT ? (double)__half2float(__ushort_as_half(hv)) : (double)qv;
    const double kap = (double)M[i] * (double)k[i];  // exact
    const double p = V * kap;
    const double e = fma(V, kap, -p);  // V kap = p + e exactly
    double t, d1, d2;
    two_sum(s, p, t, d1);
    two_sum(t, e, s, d2);
    c += d1 + d2;
    mag += fabs(p);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const double s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const double c2 = __shfl_xor_sync(0xffffffffu, c, o);
    const double m2 = __shfl_xor_sync(0xffffffffu, mag, o);
    double t, d;
    two_sum(s, s2, t, d);
    s = t;
    c = (c + c2) + d;
    mag += m2;
  }
  // |exact - (s + c)| <= 2^-88 sum |p| (each addition into c errs by at most
  // 2^-53 of a sum of |d| values, and every |d| is at most 2^-53 of the
  // running magnitude; 2^-88 covers 2 D + 10 such additions with margin)
  const double eps = mag * 3.2311742677852644e-27;  // 2^-88
  float P;
  if (!(fabs(s) <= 1.7976931348623157e308) || !(fabs(c) <= 1.7976931348623157e308)) {
    P = (float)(s + c);
  } else if (mag == 0.0) {
    P = 0.0f;  // every term is zero (e.g. a column whose codes are all 0): +0
  } else {
    const float flo = __double2float_rn(__dadd_rd(s, __dsub_rd(c, eps)));
    const float fhi = __double2float_rn(__dadd_ru(s, __dadd_ru(c, eps)));
    if (__float_as_uint(flo) == __float_as_uint(fhi)) {
      P = flo;
    } else {
      // on (or within 2^-88 of) a rounding boundary: the fixed-point sum
      P = lane == 0 ? exact_column<D>(rec, row_off, row_code, kc, rec_cap, M, k, j) : 0.0f;
      P = __shfl_sync(0xffffffffu, P, 0);
    }
  }
  return P;
}

// ------------------------------------------------------------- producer
// Issue tile x into a stage of the packed step (layout PStage). All-pivot
// heads are not staged: their record is read and written in place in the
// pool (the L2 warmed by a bulk prefetch).
template <int D>
__device__ __forceinline__ void issue_pstage(const StepArgs& a, const TileScalars& x, uint8_t* stage_base,
                                             uint64_t* bar) {
  PStage<D> s{stage_base};
  TileHdr* hd = s.hdr();
  hd->tile = x.b * a.h_v + x.h;
  if (x.slot < 0 || x.slot >= a.n_slots) {
    hd->valid = 0;
    mbar_arrive(bar);
    return;
  }
  const int b = x.b, h = x.h;
  const int hk = h / (a.h_v / a.h_k);
  const uint32_t vec = 4u * D;
  const bool kda = a.gate_kind != 0;
  const bool direct = x.kind == ROW_PIVOT;
  const bool mixed = x.kind == 0;
  uint8_t* rec_src = a.pool + (uint64_t)x.slot * a.slot_bytes + x.rec_off;
  hd->dst = rec_src;
  hd->bytes = x.rec_bytes;
  hd->valid = 1;
  hd->beta = x.beta;
  hd->g = x.g;
  hd->kind = x.kind;
  uint32_t tx = 3u * vec + (kda ? vec : 0u) + 3u * D + (mixed ? (uint32_t)D : 0u);
  if (b == 0 && h == 0) tx += a.test_extra_tx;  // testing only: this stage never completes
  if (!direct) tx += x.rec_bytes;
  mbar_arrive_expect_tx(bar, tx);
  if (direct)
    bulk_prefetch_l2(rec_src, x.rec_bytes);
  else
    bulk_g2s(s.rec(), rec_src, x.rec_bytes, bar);
  bulk_g2s(s.k(), a.k + ((size_t)b * a.h_k + hk) * D, vec, bar);
  bulk_g2s(s.q(), a.q + ((size_t)b * a.h_k + hk) * D, vec, bar);
  if (kda) bulk_g2s(s.g(), a.g + ((size_t)b * a.h_v + h) * D, vec, bar);
  bulk_g2s(s.phi(), a.t.phi + (size_t)h * D, vec, bar);
  bulk_g2s(s.row_off(), a.t.row_off + (size_t)h * D, 2u * D, bar);
  bulk_g2s(s.row_code(), a.t.row_code + (size_t)h * D, (uint32_t)D, bar);
  if (mixed) bulk_g2s(s.row_perm(), a.t.row_perm + (size_t)h * D, (uint32_t)D, bar);
}

// Thread 0: issue the next tile into stage s (or mark the stage as the end
// of the work), then start fetching the scalars of the tile after it.
template <int D>
__device__ __forceinline__ void pissue_next(const StepArgs& a, Producer* pr, uint8_t* stages, uint64_t* bars, int s,
                                            int& ahead) {
  uint8_t* base = stages + (size_t)s * a.stage_bytes;
  const int m = pr->next;
  if (m < 0) {
    PStage<D>{base}.hdr()->tile = -1;
    return;
  }
  cp_async_wait_all();
  const int k = pr->buf;
  TileScalars x;
  x.h = m / a.B;
  x.b = m - x.h * a.B;
  x.tile = x.b * a.h_v + x.h;
  x.slot = pr->slot[k];
  x.rec_off = pr->rec_off[k];
  x.rec_bytes = pr->rec_bytes[k];
  x.kind = (int)((pr->kind_word[k] >> (8 * (x.h & 3))) & 0xFFu);
  x.beta = pr->beta[k];
  x.g = a.gate_kind == 0 ? pr->g[k] : 0.0f;
  int nm = m + 1;
  if (nm >= pr->end) {
    const int n_tiles = a.B * a.h_v;
    const int n_chunks = (n_tiles + a.chunk - 1) / a.chunk;
    const int c = ahead;  // claimed a chunk ago
    if (c < n_chunks) {
      nm = c * a.chunk;
      pr->end = min(nm + a.chunk, n_tiles);
      ahead = (int)atomicAdd(a.t.sched, 1u);
    } else {
      nm = -1;
    }
  }
  pr->next = nm;
  pr->buf = k ^ 1;
  prefetch_scalars(a, pr, nm, k ^ 1);
  issue_pstage<D>(a, x, base, &bars[s]);
}

template <int D>
__device__ __forceinline__ void refill_stage_pending(const StepArgs& a, Producer* pr, uint8_t* stages, uint64_t* bars,
                                                int& ahead) {
  const int s = pr->pend;
  if (s < 0) return;
  pr->pend = -1;
  bulk_wait_read_all();
  pissue_next<D>(a, pr, stages, bars, s, ahead);
}

// ------------------------------------------------------------ pass A
// Weights of the error bound of one row (see ptile): with c the row's code
// offset, hmax the largest |h| its fp64 views take and qm the largest
// |code| (pivot rows: c = 0 and hmax = qm = the row's largest |V|), the fp64
// total of a column differs from the exact sum by at most
//   2^-53 (1 + 2^-20) sum_i (2 RPT c_i + RPT hmax_i + (NG - 1) qm_i) |M_i k_i|.
template <int D>
__device__ __forceinline__ double bound_weight(int code, float vmax) {
  using G = PGeo<D>;
  if (code == ROW_PIVOT) return (double)(G::RPT + G::NG - 1) * (double)vmax;
  const int E = code == 8 ? 12 : code;
  const double c = (double)((1 << E) + (1 << (code - 1)));
  const double hmax = (double)((1 << E) + (1 << code));
  const double qm = (double)((1 << (code - 1)) - 1);
  return 2.0 * G::RPT * c + (double)G::RPT * hmax + (double)(G::NG - 1) * qm;
}

// One row's 16 fp64 views (high words) for pass A, by width; pivot rows also
// give the largest |V| of the chunk.
template <int B, bool GLOBAL, bool VEC>
__device__ __forceinline__ void row_hi(const uint8_t* row, int cc, uint32_t (&xh)[16], float& vmax) {
  if constexpr (B == 16) {
    uint32_t w[8];
    chunk_words<16, GLOBAL, VEC>(row, cc, w);
    float mx = 0.0f;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
      xh[2 * p] = (uint32_t)__double2hiint((double)x.x);
      xh[2 * p + 1] = (uint32_t)__double2hiint((double)x.y);
      mx = fmax_nan(mx, fmax_nan(fabsf(x.x), fabsf(x.y)));
    }
    vmax = mx;
  } else {
    uint32_t w[B / 2];
    chunk_words<B, GLOBAL, VEC>(row, cc, w);
#pragma unroll
    for (int j = 0; j < 16; ++j) xh[j] = field_hi<B>(w, j);
    vmax = 0.0f;
  }
}

// -------------------------------------------------------------- pass B
// 16 codes of width B (2, 4 or 6) as floats, reading most fields where they
// lie: a field at bit s (s + B <= 23) of a source word X becomes the float
// 2^23 + f 2^s by one AND-OR (X & (mask << s) | bits of 2^23), and one
// f32x2 fma per pair, x 2^-s - (2^(23-s) + 2^(B-1)), gives the code exactly
// (every intermediate is an integer below 2^24). The source words are the
// chunk's words and a few shifts of them, chosen so that only two
// (s, s') patterns occur among the pairs.
template <int B>
__device__ __forceinline__ uint32_t magic_at(uint32_t x, int s) {
  return 0x4B000000u | (x & (((1u << B) - 1u) << s));
}
template <int B>
__device__ __forceinline__ float2 code_pair(uint32_t x0, int s0, uint32_t x1, int s1) {
  const float2 m = make_float2(__uint_as_float(magic_at<B>(x0, s0)), __uint_as_float(magic_at<B>(x1, s1)));
  const float2 k = make_float2(1.0f / (float)(1u << s0), 1.0f / (float)(1u << s1));
  const float2 c = make_float2(-(float)((1u << (23 - s0)) + (1u << (B - 1))),
                               -(float)((1u << (23 - s1)) + (1u << (B - 1))));
  return __ffma2_rn(m, k, c);
}
template <int B>
__device__ __forceinline__ void unpack16_inplace(const uint32_t (&w)[B / 2], float2 (&V)[8]) {
  if constexpr (B == 6) {
    // 24-bit groups g (fields 4g .. 4g+3 at 0, 6, 12, 18); the field at 18
    // comes from a second shift, at 6
    const uint32_t G[4] = {w[0], __funnelshift_r(w[0], w[1], 24), __funnelshift_r(w[1], w[2], 16), w[2] >> 8};
    const uint32_t H[4] = {w[0] >> 12, w[1] >> 4, __funnelshift_r(w[1], w[2], 28), w[2] >> 20};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      V[2 * g] = code_pair<6>(G[g], 0, G[g], 6);
      V[2 * g + 1] = code_pair<6>(G[g], 12, H[g], 6);
    }
  } else if constexpr (B == 4) {
    // per word: fields 0..3 at 0, 4, 8, 12 and fields 4..7 at the same
    // places of the word shifted by 16
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t Y = w[k] >> 16;
      V[4 * k] = code_pair<4>(w[k], 0, w[k], 4);
      V[4 * k + 1] = code_pair<4>(w[k], 8, w[k], 12);
      V[4 * k + 2] = code_pair<4>(Y, 0, Y, 4);
      V[4 * k + 3] = code_pair<4>(Y, 8, Y, 12);
    }
  } else {
    static_assert(B == 2, "widths 2, 4, 6");
    // X_k = w >> 4k holds fields 2k, 2k+1 at 0, 2 and 2k+8, 2k+9 at 16, 18
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t X = w[0] >> (4 * k);
      V[k] = code_pair<2>(X, 0, X, 2);
      V[4 + k] = code_pair<2>(X, 16, X, 18);
    }
  }
}

// One row's 16 stored values as floats (codes, or fp16 values).
template <int B, bool GLOBAL, bool VEC>
__device__ __forceinline__ void row_values(const uint8_t* row, int cc, float2 (&V)[8]) {
  if constexpr (B == 16) {
    uint32_t w[8];
    chunk_words<16, GLOBAL, VEC>(row, cc, w);
#pragma unroll
    for (int p = 0; p < 8; ++p) V[p] = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
  } else if constexpr (B == 8) {
    uint32_t w[4];
    chunk_words<8, GLOBAL, VEC>(row, cc, w);
    const float2 off = f2(-(8388608.0f + 128.0f));
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t x = w[p >> 1];
      const int j = 2 * (p & 1);
      const float2 m = make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650u | (uint32_t)j)),
                                   __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650u | (uint32_t)(j + 1))));
      V[p] = __fadd2_rn(m, off);
    }
  } else {
    uint32_t w[B / 2];
    chunk_words<B, GLOBAL, VEC>(row, cc, w);
    unpack16_inplace<B>(w, V);
  }
}

// Row maximum of |T'| over the LPR lanes of a row (NaN if any is NaN).
template <int D>
__device__ __forceinline__ float prow_absmax(const float2 (&t)[8]) {
  const float a0 = absmax3_nan(t[0].x, t[0].y, t[1].x);
  const float a1 = absmax3_nan(t[1].y, t[2].x, t[2].y);
  const float a2 = absmax3_nan(t[3].x, t[3].y, t[4].x);
  const float a3 = absmax3_nan(t[4].y, t[5].x, t[5].y);
  const float a4 = absmax3_nan(t[6].x, t[6].y, t[7].x);
  const float b0 = absmax3_nan(a0, a1, a2);
  const float b1 = absmax3_nan(a3, a4, t[7].y);
  float x = fmax_nan(b0, b1);
#pragma unroll
  for (int s = 1; s < PGeo<D>::LPR; s <<= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, s));
  return x;
}

// Requantize the QS rows of group grp (row slots (grp QS + u) NG + rg):
// one lane per row of the group computes the row scale, the others take it
// by shuffle; new codes (or fp16 pivots) written into the record. A row
// holding a NaN gets scale 0 and all codes 0 (status bit NaN).
template <int D, int KC, bool DIRECT>
__device__ __forceinline__ uint32_t prequant(uint8_t* rec, const uint16_t* row_off, const uint8_t* row_code,
                                             const uint8_t* row_perm, const float* phi, uint32_t rec_cap, int grp,
                                             int rg, int cc, const float2 (&T)[PGeo<D>::QS][8]) {
  using G = PGeo<D>;
  constexpr int QS = G::QS;
  uint32_t st = 0;
  auto row_of = [&](int u) -> int {
    const int s = (grp * QS + u) * G::NG + rg;
    return KC ? s : (row_perm[s] & (D - 1));
  };
  auto row_ptr = [&](int i) -> uint8_t* {
    if constexpr (KC != 0) {
      constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
      return rec + 2u * D + (uint32_t)i * rb;
    } else {
      return rec + min((uint32_t)row_off[i], rec_cap);
    }
  };
  if constexpr (KC == ROW_PIVOT) {
#pragma unroll
    for (int u = 0; u < QS; ++u) st |= store_row_pivot<DIRECT>(row_ptr(row_of(u)), cc, T[u]);
    return st;
  } else {
    float m[QS];
#pragma unroll
    for (int u = 0; u < QS; ++u) m[u] = prow_absmax<D>(T[u]);
    const int mine = cc % QS;
    float mm = m[0];
#pragma unroll
    for (int u = 1; u < QS; ++u) mm = mine == u ? m[u] : mm;
    const int im = row_of(mine);
    const int cm = KC ? KC : row_code[im];
    // A row holding a NaN keeps ir = lim = 0: every T' then clamps to +-0 (a
    // NaN too: min.xorsign.abs returns its other operand) and rounds to code
    // 0, with row scale 0.
    float ir_m = 0.0f, lim_m = 0.0f;
    if (cm != ROW_PIVOT) {
      uint16_t rbits = 0;
      if (mm != mm) st |= ST_NAN;
      if (mm == mm) {
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
        lim_m = __fmul_rn(qm, R);  // qmax r', exact
        rbits = __half_as_ushort(rh);
      }
      if (cc < QS) reinterpret_cast<uint16_t*>(rec)[im] = rbits;
    }
    const int base = (int)(threadIdx.x & 31) - cc;
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      const float ir = __shfl_sync(0xffffffffu, ir_m, base + u);
      const float lim = __shfl_sync(0xffffffffu, lim_m, base + u);
      const int i = row_of(u);
      const int code = KC ? KC : row_code[i];
      uint8_t* row = row_ptr(i);
      if (code == ROW_PIVOT) {
        st |= store_row_pivot<false>(row, cc, T[u]);
      } else if constexpr (KC != 0) {
        store_row_q<KC>(row, cc, ir, lim, T[u]);
      } else {
        switch (code) {
          case 8: store_row_q<8>(row, cc, ir, lim, T[u]); break;
          case 6: store_row_q<6>(row, cc, ir, lim, T[u]); break;
          case 4: store_row_q<4>(row, cc, ir, lim, T[u]); break;
          default: store_row_q<2>(row, cc, ir, lim, T[u]); break;
        }
      }
    }
    return st;
  }
}

// fp64 deposit of a thread's 16 column partials (16-byte pieces rotated by
// cc so that the lanes of a row group write different banks).
template <int D>
__device__ __forceinline__ void pdeposit_f64(double* red, int rg, int cc, const double (&acc)[16]) {
#pragma unroll
  for (int p = 0; p < 8; ++p)
    *reinterpret_cast<double2*>(red + rg * D + 16 * cc + 2 * (p ^ (cc & 7))) = make_double2(acc[2 * p], acc[2 * p + 1]);
}
template <int D>
__device__ __forceinline__ double ptotal_f64(const double* red, int j) {
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 2 * ((e >> 1) ^ (cj & 7)) + (e & 1);
  double a[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int g = 0; g < PGeo<D>::NG; ++g) a[g & 3] += red[g * D + off];
  return (a[0] + a[1]) + (a[2] + a[3]);
}
// fp32 deposit and total of the o partials (same rotation, 16-byte pieces
// of four floats).
template <int D>
__device__ __forceinline__ void pdeposit_f32(float* red, int rg, int cc, const float2 (&part)[8]) {
  const int sw = cc & 3;
#pragma unroll
  for (int p = 0; p < 4; ++p)
    *reinterpret_cast<float4*>(red + rg * D + 16 * cc + 4 * (p ^ sw)) =
        make_float4(part[2 * p].x, part[2 * p].y, part[2 * p + 1].x, part[2 * p + 1].y);
}
template <int D>
__device__ __forceinline__ float ptotal_f32(const float* red, int j) {
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 4 * ((e >> 2) ^ (cj & 3)) + (e & 3);
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < PGeo<D>::NG; ++g) a[g & 3] = __fadd_rn(a[g & 3], red[g * D + off]);
  return __fadd_rn(__fadd_rn(a[0], a[1]), __fadd_rn(a[2], a[3]));
}

// ------------------------------------------------------------ one tile
// KC: width shared by every row of the head (ROW_PIVOT: all-pivot head, read
// and written in place in the pool), or 0 for a head whose rows differ.
// Returns false when a bounded wait gave up (the tile is abandoned: pass A
// still runs, on stale shared memory, before the decision at B1; row
// offsets of mixed-width heads are clamped to rec_cap, and a stage keeps
// 2 D bytes after the record, so a row read of any width stays inside the
// stage whatever the tables hold). The
// loops over a thread's rows are not unrolled (per-row scalars come by
// shuffle or from shared memory), which keeps each width's code small
// enough for the instruction cache.
template <int D, int KC>
__device__ __forceinline__ bool ptile(const StepArgs& a, const PStage<D>& S, int sidx, uint32_t parity, int n,
                                      uint64_t* bars, uint64_t* free_bar, uint8_t* stages, uint8_t* red, float* wsh,
                                      float* msh, double* eps_sh, int* abort_sh, Producer* pr, int& ahead, int rg,
                                      int cc, uint32_t& st) {
  using G = PGeo<D>;
  constexpr bool DIRECT = KC == ROW_PIVOT;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int base = lane - cc;
  const bool kda = a.gate_kind != 0;
  const TileHdr* hd = S.hdr();
  const int tile = hd->tile;
  const int h = tile % a.h_v;
  uint8_t* rec = DIRECT ? hd->dst : S.rec();
  double* red64 = reinterpret_cast<double*>(red);

  // per-column inputs of the column this thread totals (column tid)
  const float cj = __ldg(a.t.col + (size_t)h * D + tid);
  const float icj = __ldg(a.t.icol + (size_t)h * D + tid);
  const float vj = __ldg(a.v + (size_t)tile * D + tid);

  if (!mbar_wait_bounded(&bars[sidx], parity, a.wait_ns)) *abort_sh = 1;

  // ---- row factors: lane cc handles row slot cc of its row group:
  // M = fp32(r g) (quantized row) or g (pivot row); kap = M k exactly in fp64
  const uint16_t* rt_off = S.row_off();
  const uint8_t* rt_code = S.row_code();
  const uint8_t* rt_perm = S.row_perm();
  const int sm = cc * G::NG + rg;
  const int im = KC ? sm : (rt_perm[sm] & (D - 1));
  const int cm = KC ? KC : rt_code[im];
  const float gm = kda ? S.g()[im] : hd->g;
  const float Mm = cm == ROW_PIVOT ? gm : __fmul_rn(__half2float(reinterpret_cast<const __half*>(rec)[im]), gm);
  msh[im] = Mm;
  const double kapm = (double)Mm * (double)S.k()[im];
  // the bias of the fp64 views of this thread's rows, sum_r c_r kap_r (the
  // RPT rows of a thread are the rows of its row group's lanes)
  double off = cm == ROW_PIVOT ? 0.0 : code_offset(cm) * kapm;
#pragma unroll
  for (int o = 1; o < G::LPR; o <<= 1) off += __shfl_xor_sync(0xffffffffu, off, o);

  // ---- pass A: fp64 partials of S^T k over this thread's rows
  float vm = 0.0f;  // pivot rows: largest |V| of row slot cc (for the bound)
  double acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = -off;
#pragma unroll 1
  for (int r = 0; r < G::RPT; ++r) {
    const int s = r * G::NG + rg;
    const double kap = __shfl_sync(0xffffffffu, kapm, base + r);
    uint32_t xh[16];
    float vmax;
    if constexpr (KC != 0) {
      constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
      row_hi<KC == ROW_PIVOT ? 16 : KC, DIRECT, true>(rec + 2u * D + (uint32_t)s * rb, cc, xh, vmax);
    } else {
      const int i = rt_perm[s] & (D - 1);
      const uint8_t* row = rec + min((uint32_t)rt_off[i], a.rec_cap);
      switch (rt_code[i]) {
        case 8: row_hi<8, false, false>(row, cc, xh, vmax); break;
        case 6: row_hi<6, false, false>(row, cc, xh, vmax); break;
        case 4: row_hi<4, false, false>(row, cc, xh, vmax); break;
        case 2: row_hi<2, false, false>(row, cc, xh, vmax); break;
        default: row_hi<16, false, false>(row, cc, xh, vmax); break;
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = fma(__hiloint2double((int)xh[j], 0), kap, acc[j]);
    if (KC == ROW_PIVOT || KC == 0) {
#pragma unroll
      for (int o = 1; o < G::LPR; o <<= 1) vmax = fmax_nan(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      if (cc == r) vm = vmax;
    }
  }
  // the buffer is free once every thread has read the previous tile's o partials
  bool free_ok = true;
  if (n > 0) free_ok = mbar_wait_bounded(free_bar, (uint32_t)(n - 1) & 1u, a.wait_ns);
  if (free_ok) pdeposit_f64<D>(red64, rg, cc, acc);
  else *abort_sh = 1;

  // ---- the tile's error bound: lane cc adds row slot cc's weight
  {
    double e = bound_weight<D>(cm, vm) * fabs(kapm);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    if (lane == 0) eps_sh[tid >> 5] = e;
  }
  __syncthreads();  // B1: the S^T k partials and the bound are complete
  if (*abort_sh) return false;
  if (tid == 0) refill_stage_pending<D>(a, pr, stages, bars, ahead);

  // ---- column total, certified rounding, w
  {
    const double t = ptotal_f64<D>(red64, tid);
    double eb = 0.0;
#pragma unroll
    for (int w = 0; w < G::NW; ++w) eb += eps_sh[w];
    const double eps = eb * 1.1102230246251566e-16 * (1.0 + 9.5367431640625e-7);  // 2^-53 (1 + 2^-20)
    float P = 0.0f;
    bool redo = false;
    if (!(fabs(t) <= 1.7976931348623157e308)) {
      P = (float)t;  // NaN or inf among the terms: the IEEE result
    } else if (eps == 0.0) {
      P = 0.0f;  // every term is zero
    } else {
      const float flo = __double2float_rn(__dsub_rd(t, eps));
      const float fhi = __double2float_rn(__dadd_ru(t, eps));
      P = flo;
      redo = __float_as_uint(flo) != __float_as_uint(fhi);
    }
    // columns the bound could not round: again, by the whole warp
    uint32_t todo = __ballot_sync(0xffffffffu, redo);
    if (todo && lane == 0) atomicAdd(a.t.xcount, (uint32_t)__popc(todo));
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const float Px = column_warp<D>(rec, rt_off, rt_code, KC, a.rec_cap, msh, S.k(), (tid & ~31) + src);
      if (lane == src) P = Px;
    }
    const float p = __fmul_rn(cj, P);
    const float u = __fmul_rn(hd->beta, __fsub_rn(vj, p));
    wsh[tid] = __fmul_rn(u, icj);
  }
  __syncthreads();  // B2: w is complete

  // ---- pass B: update (one rounding), o partials, requantization
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
  float2 part[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) part[p] = make_float2(0.0f, 0.0f);
#pragma unroll 1
  for (int grp = 0; grp < G::RPT / G::QS; ++grp) {
    float2 T[G::QS][8];
#pragma unroll
    for (int u = 0; u < G::QS; ++u) {
      const int s = (grp * G::QS + u) * G::NG + rg;
      const int i = KC ? s : (rt_perm[s] & (D - 1));
      float2 V[8];
      if constexpr (KC != 0) {
        constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
        row_values<KC == ROW_PIVOT ? 16 : KC, DIRECT, true>(rec + 2u * D + (uint32_t)i * rb, cc, V);
      } else {
        const uint8_t* row = rec + min((uint32_t)rt_off[i], a.rec_cap);
        switch (rt_code[i]) {
          case 8: row_values<8, false, false>(row, cc, V); break;
          case 6: row_values<6, false, false>(row, cc, V); break;
          case 4: row_values<4, false, false>(row, cc, V); break;
          case 2: row_values<2, false, false>(row, cc, V); break;
          default: row_values<16, false, false>(row, cc, V); break;
        }
      }
      const float kr = S.k()[i], qr = S.q()[i], M = msh[i];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        T[u][p] = __ffma2_rn(V[p], f2(M), __fmul2_rn(f2(kr), W[p]));
        part[p] = __ffma2_rn(T[u][p], f2(qr), part[p]);
      }
    }
    st |= prequant<D, KC, DIRECT>(rec, rt_off, rt_code, rt_perm, S.phi(), a.rec_cap, grp, rg, cc, T);
  }
  pdeposit_f32<D>(reinterpret_cast<float*>(red), rg, cc, part);
  if (!DIRECT) fence_proxy_async_smem();  // the new record is read by the bulk store
  __syncthreads();  // B3: the o partials and the new record are complete

  {
    const float O = ptotal_f32<D>(reinterpret_cast<const float*>(red), tid);
    const float oj = __fmul_rn(cj, O);
    if (oj != oj) st |= ST_NAN;
    a.o[(size_t)tile * D + tid] = oj;
  }
  mbar_arrive(free_bar);  // this thread is done with the o partials
  if (tid == 0) {
    if (!DIRECT) {
      bulk_s2g(hd->dst, S.rec(), hd->bytes);
      bulk_commit();
    }
    pr->pend = sidx;
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(PGeo<D>::NT, 4) k_decode_step_packed(const StepArgs a) {
  using G = PGeo<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[kPackedStages];
  __shared__ __align__(8) uint64_t free_bar;
  __shared__ __align__(16) float wsh[D];
  __shared__ __align__(16) float msh[D];
  __shared__ double eps_sh[G::NW];
  __shared__ Producer prod;
  __shared__ uint32_t st_sh;
  __shared__ int abort_sh;
  // [S^T k (fp64) / o (fp32) partials: NG D 8 bytes][stage 0][stage 1]
  uint8_t* red = smem;
  uint8_t* stages = smem + (size_t)G::NG * D * 8;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int cc = lane % G::LPR;
  const int rg = warp * G::RPW + lane / G::LPR;

  int ahead = 0;  // thread 0: the chunk claimed for after the current one
  if (tid == 0) {
    for (int s = 0; s < a.nstage; ++s) mbar_init(&bars[s], 1);
    mbar_init(&free_bar, G::NT);
    fence_mbar_init();
    st_sh = 0;
    abort_sh = 0;
    producer_start(a, &prod, ahead);
    for (int s = 0; s < a.nstage; ++s) pissue_next<D>(a, &prod, stages, bars, s, ahead);
  }
  __syncthreads();

  uint32_t st = 0;
  int n = 0;
  for (;; ++n) {
    const int sidx = n % a.nstage;
    const uint32_t parity = (uint32_t)(n / a.nstage) & 1u;
    const PStage<D> S{stages + (size_t)sidx * a.stage_bytes};
    // The header was written by thread 0 before at least one block barrier
    // that every thread has passed since, so it is read without waiting for
    // the stage's data; the control flow below is uniform over the CTA.
    const int tile = S.hdr()->tile;  // b * h_v + h
    if (tile < 0) break;
    if (!S.hdr()->valid) {
      a.o[(size_t)tile * D + tid] = 0.0f;
      st |= ST_SLOT;
      __syncthreads();  // every thread has read the header and finished the previous tile
      mbar_arrive(&free_bar);
      if (tid == 0) {
        refill_stage_pending<D>(a, &prod, stages, bars, ahead);
        prod.pend = sidx;  // nothing was loaded or stored: refill at the next refill point
      }
      __syncthreads();  // publish the refilled header before its tile is read
      continue;
    }
    bool ok;
    switch (S.hdr()->kind) {
      case 8:
        ok = ptile<D, 8>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh, &prod,
                         ahead, rg, cc, st);
        break;
      case 6:
        ok = ptile<D, 6>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh, &prod,
                         ahead, rg, cc, st);
        break;
      case 4:
        ok = ptile<D, 4>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh, &prod,
                         ahead, rg, cc, st);
        break;
      case 2:
        ok = ptile<D, 2>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh, &prod,
                         ahead, rg, cc, st);
        break;
      case ROW_PIVOT:
        ok = ptile<D, ROW_PIVOT>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh,
                                 &prod, ahead, rg, cc, st);
        break;
      default:
        ok = ptile<D, 0>(a, S, sidx, parity, n, bars, &free_bar, stages, red, wsh, msh, eps_sh, &abort_sh, &prod,
                         ahead, rg, cc, st);
        break;
    }
    if (!ok) {
      st |= ST_TIMEOUT;
      break;
    }
  }
  if (st) atomicOr(&st_sh, st);
  __syncthreads();
  if (tid == 0) {
    if (abort_sh) {
      // let the loads still in flight land before the CTA exits: every
      // issued stage whose wait has not completed gets a bounded wait
      for (int k = 0; k < a.nstage; ++k) {
        const TileHdr* hd = PStage<D>{stages + (size_t)((n + k) % a.nstage) * a.stage_bytes}.hdr();
        if (hd->tile >= 0 && hd->valid)
          (void)mbar_wait_bounded(&bars[(n + k) % a.nstage], (uint32_t)((n + k) / a.nstage) & 1u, a.wait_ns);
      }
    }
    bulk_wait_all();
    if (st_sh) atomicOr(a.t.status, st_sh);
    // The last CTA to finish resets the chunk counter for the next launch
    // (every CTA's claims are ordered before its count by the fence).
    __threadfence();
    if (atomicAdd(a.t.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(a.t.sched, 0u);
      atomicExch(a.t.sched + 1, 0u);
    }
  }
}

}  // namespace sqk
