// sq_window.cuh -- one token of the per-window variant on a packed state pool
// (sm_100a).
//
// Per-window quantization ("线性注意力每生成一个token都要搬状态，LeapQuant把它压到
// 8位还不掉点" (wink.run), the first of its three techniques): the packed state
// of a (request, value head) tile stays frozen for a window of W tokens; each
// token's key k_tau, update vector u_tau and gate G_tau go to a high-precision
// buffer (fp32, one window record per tile); the token's outputs come from
// the frozen state and the buffer together; when the window is full the state
// is requantized once and the buffer is emptied.
//
// For a tile whose buffer holds n tokens (the current token is token n; its
// gate is G_n):
//   E_tau,i = prod_{sigma = tau+1 .. n} G_sigma,i            (tau = -1 .. n-1)
//   S_ij    = E_-1,i S0_ij + sum_{tau<n} E_tau,i k_tau,i u_tau,j   (gated, before
//             token n's delta), S0_ij = V_ij M_i c_j the frozen state
//   p_j = sum_i S_ij k_i = c_j sum_i V_ij a_i + sum_tau alpha_tau u_tau,j,
//         a_i = E_-1,i M_i k_i,  alpha_tau = sum_i E_tau,i k_tau,i k_i
//   u_j = fp32(beta (v_j - p_j))
//   o_j = sum_i (S_ij + k_i u_j) q_i
//       = c_j sum_i V_ij b_i + sum_tau gamma_tau u_tau,j + (k . q) u_j,
//         b_i = E_-1,i M_i q_i,  gamma_tau = sum_i E_tau,i k_tau,i q_i
// so a token reads the packed codes once and forms two fp64 column sums of
// them, reads the buffer's n rows, appends its own row, and writes nothing
// of the state. When the window is full the state is formed in the record's
// column-normalised units and in fp32, the way the step forms T':
//   T_ij = fmaf(V_ij, a_i, t_ij),  t_ij = fmaf(e_tau,i, w_tau,j, t_ij) over the
//   W tokens in order from t = 0,  a_i = fp32(E_-1,i M_i),
//   e_tau,i = fp32(E_tau,i k_tau,i) (E = 1 for the last token),
//   w_tau,j = fp32(u_tau,j fp32(1/c_j))
// (a rank-W update of the frozen state), and requantized in place by the
// step's rules (row scales from the row maximum and the clip ratio,
// round-up to fp16, codes rounded to nearest even).
//
// Work distribution. Persistent CTAs: four consumer warps in the packed
// step's thread map (PGeo: a thread owns 16 columns of RPT key rows) and one
// producer warp. Tiles are taken in head-major order, tile m of the launch
// going to CTA m mod grid. The producer's lane 0 reads each tile's scalars
// one tile ahead (slot, window count, beta, gate), and fills one of two
// stages with 1-D bulk copies (cp.async.bulk, no multicast) completed on an
// mbarrier: q, k, v, the KDA gate vector, the head's column scales and row
// tables, and the n buffered key, u and gate rows; it also asks L2 to
// prefetch the tile's packed record, which the consumers then read from
// global memory (they write it in place at the end of a window). A stage is
// released by the first consumer barrier of the tile after it.
#pragma once

#include "sq_step.cuh"

namespace sqk {

constexpr uint32_t ST_WINDOW = 16u;  // a window record's count was outside [0, W)

struct WindowArgs {
  uint8_t* pool;
  uint8_t* wbuf;          // [n_slots][h_v] window records
  const float* q;         // [B, h_k, d]
  const float* k;         // [B, h_k, d]
  const float* v;         // [B, h_v, d]
  const float* beta;      // [B, h_v]
  const float* g;         // [B, h_v] or [B, h_v, d]
  float* o;               // [B, h_v, d]
  const int32_t* slots;   // [B] or null
  int32_t B, h_v, h_k, n_slots, gate_kind, W;
  uint64_t slot_bytes;
  uint64_t wait_ns;       // limit of every bounded wait
  uint32_t wrec_bytes;    // bytes of one window record
  Tables t;
};

// Header of a stage, written by the producer before the stage's mbarrier
// phase completes.
struct WHdr {
  uint8_t* rec;    // the tile's packed record (pool)
  uint8_t* wrec;   // the tile's window record
  uint32_t bytes;  // record bytes
  int32_t tile;    // b h_v + h, or -1: no more tiles
  int32_t valid;   // 1: a tile to compute; 0: slot id out of range; 2: window count out of range
  int32_t n;       // buffered tokens
  int32_t kind;    // width shared by the head's rows (ROW_PIVOT: all pivot), 0: mixed
  float beta, g;
};

// Stage layout (bytes): [hdr 64][q][k][v][g][col][icol] (fp32, d each)
// [row_off u16 d][row_code d][row_perm d][k rows fp32 (W-1) d][u rows fp32 (W-1) d]
// [gates fp32 (W-1) gd, padded to 16 B], padded to 128 B. At a window's end
// the k rows are replaced by e rows and the u rows by w rows. Then, after
// both stages, the work area: [S^T k partials fp64 NW d][S^T q partials fp64
// NW d][E k products fp64 (W-1) d][a][b][k][q][E_-1] (fp64 d each)
// [M][u or w][a][e of the current token] (fp32 d each)[alpha, gamma fp64 W
// each, k.q, pad].
struct WLay {
  uint32_t q, k, v, g, col, icol, roff, rcode, rperm, kb, ub, gb, stage;
  uint32_t redp, redo, ek, a, b, kd, qd, d0, m, un, af, ecur, ag, total;
};
__host__ __device__ inline uint32_t wround(uint32_t x, uint32_t m) { return (x + m - 1) / m * m; }
__host__ __device__ inline WLay window_layout(int D, int W, int gd) {
  WLay L;
  const uint32_t d = (uint32_t)D, w1 = (uint32_t)(W - 1);
  L.q = 64;
  L.k = L.q + 4 * d;
  L.v = L.k + 4 * d;
  L.g = L.v + 4 * d;
  L.col = L.g + 4 * d;
  L.icol = L.col + 4 * d;
  L.roff = L.icol + 4 * d;
  L.rcode = L.roff + 2 * d;
  L.rperm = L.rcode + d;
  L.kb = L.rperm + d;
  L.ub = L.kb + 4 * w1 * d;
  L.gb = L.ub + 4 * w1 * d;
  L.stage = wround(L.gb + 4 * wround(w1 * (uint32_t)gd, 4), 128);
  const uint32_t nw = (uint32_t)D / 32;  // consumer warps (PGeo: D threads)
  L.redp = 2 * L.stage;
  L.redo = L.redp + 8 * nw * d;
  L.ek = L.redo + 8 * nw * d;
  L.a = L.ek + 8 * (w1 > 0 ? w1 : 1) * d;
  L.b = L.a + 8 * d;
  L.kd = L.b + 8 * d;
  L.qd = L.kd + 8 * d;
  L.d0 = L.qd + 8 * d;
  L.m = L.d0 + 8 * d;
  L.un = L.m + 4 * d;
  L.af = L.un + 4 * d;
  L.ecur = L.af + 4 * d;
  L.ag = L.ecur + 4 * d;
  L.total = wround(L.ag + 8 * (2 * (uint32_t)W + 2), 128);
  return L;
}

// Column sums of the 16 fp64 partials of every thread: the RPW row groups of
// a warp are added by shuffles, then the warp's lanes of row group 0 deposit
// (16-byte pieces rotated by cc against bank conflicts) and thread j adds
// the NW warps' values of column j.
template <int D>
__device__ __forceinline__ void wdeposit(double* red, int warp, int lane, int cc, double (&acc)[16]) {
  using G = PGeo<D>;
#pragma unroll
  for (int o = G::LPR; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  if (lane < G::LPR) {
#pragma unroll
    for (int p = 0; p < 8; ++p)
      *reinterpret_cast<double2*>(red + warp * D + 16 * cc + 2 * (p ^ (cc & 7))) =
          make_double2(acc[2 * p], acc[2 * p + 1]);
  }
}
template <int D>
__device__ __forceinline__ double wtotal(const double* red, int j) {
  const int cj = j >> 4, e = j & 15;
  const int off = 16 * cj + 2 * ((e >> 1) ^ (cj & 7)) + (e & 1);
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < PGeo<D>::NW; ++w) t += red[w * D + off];
  return t;
}

template <int D>
struct WGeo {
  static constexpr int NC = PGeo<D>::NT;  // consumer threads
  static constexpr int NT = NC + 32;      // plus the producer warp
};

__device__ __forceinline__ void consumer_sync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }

// Bounded wait on an mbarrier phase that suspends the thread in the
// hardware until the phase completes (or a 20 us hint runs out) instead of
// polling, so that a waiting warp takes no issue slots from the others.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_suspend(uint64_t* bar, uint32_t parity, uint64_t max_ns) {
  if (mbar_try_wait_suspend(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (true) {
    if (mbar_try_wait_suspend(bar, parity)) return true;
    uint64_t t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 > max_ns) return false;
  }
}

// The producer's view of one tile (loads issued one tile ahead of use).
struct WScal {
  int m, b, h, slot;
  uint32_t rec_off, rec_bytes;
  int kind;
  float beta, g;
};

__device__ __forceinline__ WScal wscal(const WindowArgs& a, int m) {
  WScal x;
  x.m = m;
  if (m >= a.B * a.h_v) return x;
  x.h = m / a.B;
  x.b = m - x.h * a.B;
  x.slot = a.slots ? a.slots[x.b] : x.b;
  x.rec_off = a.t.rec_off[x.h];
  x.rec_bytes = a.t.rec_bytes[x.h];
  x.kind = a.t.head_kind[x.h];
  const int tile = x.b * a.h_v + x.h;
  x.beta = a.beta[tile];
  x.g = a.gate_kind == 0 ? a.g[tile] : 0.0f;
  return x;
}
__device__ __forceinline__ bool wvalid_slot(const WindowArgs& a, const WScal& x) {
  return x.slot >= 0 && x.slot < a.n_slots;
}
__device__ __forceinline__ int wcount(const WindowArgs& a, const WScal& x) {
  if (x.m >= a.B * a.h_v || !wvalid_slot(a, x)) return 0;
  return *reinterpret_cast<const int32_t*>(a.wbuf + ((uint64_t)x.slot * a.h_v + x.h) * a.wrec_bytes);
}

template <int D>
__device__ __forceinline__ void wissue(const WindowArgs& a, const WLay& L, uint8_t* stg, uint64_t* full,
                                       const WScal& x, int n) {
  WHdr* hd = reinterpret_cast<WHdr*>(stg);
  const bool kda = a.gate_kind != 0;
  const int gd = kda ? D : 1;
  hd->tile = x.b * a.h_v + x.h;
  hd->n = n;
  if (!wvalid_slot(a, x) || n < 0 || n >= a.W) {
    hd->valid = wvalid_slot(a, x) ? 2 : 0;
    mbar_arrive(full);
    return;
  }
  const int tile = hd->tile;
  const int hk = x.h / (a.h_v / a.h_k);
  const bool mixed = x.kind == 0;
  uint8_t* rec = a.pool + (uint64_t)x.slot * a.slot_bytes + x.rec_off;
  uint8_t* wrec = a.wbuf + ((uint64_t)x.slot * a.h_v + x.h) * a.wrec_bytes;
  hd->rec = rec;
  hd->wrec = wrec;
  hd->bytes = x.rec_bytes;
  hd->valid = 1;
  hd->kind = x.kind;
  hd->beta = x.beta;
  hd->g = x.g;
  const uint32_t vec = 4u * D;
  const uint32_t rows = 4u * (uint32_t)n * D;
  const uint32_t gates = wround(4u * (uint32_t)(n * gd), 16);
  uint32_t tx = 5u * vec + (kda ? vec : 0u) + (mixed ? 4u * D : 0u);
  if (n > 0) tx += 2u * rows + gates;
  mbar_arrive_expect_tx(full, tx);
  bulk_g2s(stg + L.q, a.q + ((size_t)x.b * a.h_k + hk) * D, vec, full);
  bulk_g2s(stg + L.k, a.k + ((size_t)x.b * a.h_k + hk) * D, vec, full);
  bulk_g2s(stg + L.v, a.v + (size_t)tile * D, vec, full);
  if (kda) bulk_g2s(stg + L.g, a.g + (size_t)tile * D, vec, full);
  bulk_g2s(stg + L.col, a.t.col + (size_t)x.h * D, vec, full);
  bulk_g2s(stg + L.icol, a.t.icol + (size_t)x.h * D, vec, full);
  if (mixed) {
    bulk_g2s(stg + L.roff, a.t.row_off + (size_t)x.h * D, 2u * D, full);
    bulk_g2s(stg + L.rcode, a.t.row_code + (size_t)x.h * D, (uint32_t)D, full);
    bulk_g2s(stg + L.rperm, a.t.row_perm + (size_t)x.h * D, (uint32_t)D, full);
  }
  if (n > 0) {
    bulk_g2s(stg + L.kb, wrec + 16, rows, full);
    bulk_g2s(stg + L.ub, wrec + 16 + 4u * (uint32_t)a.W * D, rows, full);
    bulk_g2s(stg + L.gb, wrec + 16 + 8u * (uint32_t)a.W * D, gates, full);
  }
  bulk_prefetch_l2(rec, x.rec_bytes);
}

// Position of column j in a rotated w row: the four 4-column pieces of each
// 16-column chunk cj are rotated by cj / 2, so that chunk cc's piece p is at
// 4 ((p + cc / 2) mod 4).
__device__ __forceinline__ int wswz(int j) {
  const int cj = j >> 4, e = j & 15;
  return 16 * cj + 4 * (((e >> 2) + (cj >> 1)) & 3) + (e & 3);
}

// Pointers into the work area.
struct WWork {
  double* redp;
  double* redo;
  double* ek;
  double* a;
  double* b;
  double* kd;
  double* qd;
  double* d0;
  float* m;
  float* un;
  float* af;
  float* ecur;
  double* ag;
};

// One row's contribution to the two column sums: the 16 codes as fp64 views
// (high words: 2^E + field, see field_hi), times a_i into accP and b_i into
// accO; the views' offset 2^E + 2^(b-1) is taken off once per row (offP, offO).
template <int B>
__device__ __forceinline__ void wrow_q(const uint32_t* w, double ai, double bi, double (&accP)[16],
                                       double (&accO)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const double x = __hiloint2double((int)field_hi<B>(w, j), 0);
    accP[j] = fma(x, ai, accP[j]);
    accO[j] = fma(x, bi, accO[j]);
  }
}
// A pivot row: 16 fp16 values.
__device__ __forceinline__ void wrow_pivot(const uint32_t* w, double ai, double bi, double (&accP)[16],
                                           double (&accO)[16]) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
    const double x0 = (double)f.x, x1 = (double)f.y;
    accP[2 * p] = fma(x0, ai, accP[2 * p]);
    accP[2 * p + 1] = fma(x1, ai, accP[2 * p + 1]);
    accO[2 * p] = fma(x0, bi, accO[2 * p]);
    accO[2 * p + 1] = fma(x1, bi, accO[2 * p + 1]);
  }
}
// The b/2 words (quantized row) or 8 words (pivot row) of chunk cc, read from
// global memory with 4-byte loads (rows of mixed-width heads are only 4-byte
// aligned).
__device__ __forceinline__ void wload_words(const uint8_t* row, int code, int cc, uint32_t (&w)[8]) {
  const int nw = code == ROW_PIVOT ? 8 : code / 2;
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row + (code == ROW_PIVOT ? 32 : 2 * code) * cc);
#pragma unroll
  for (int x = 0; x < 8; ++x)
    if (x < nw) w[x] = p[x];
}

// The frozen pass of a head whose rows all have width KC (ROW_PIVOT: all
// pivot): the chunks of all of the thread's rows are loaded first (pivot
// heads: four rows at a time), then used.
template <int D, int KC>
__device__ __forceinline__ void wfrozen_uniform(const uint8_t* rec, const WWork& w, int rg, int cc,
                                                double (&accP)[16], double (&accO)[16]) {
  using G = PGeo<D>;
  constexpr int NWD = KC == ROW_PIVOT ? 8 : KC / 2;
  constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
  constexpr int RB = NWD <= 4 ? G::RPT : (G::RPT < 4 ? G::RPT : 4);
  static_assert(G::RPT % RB == 0, "row batches");
  double offP = 0.0, offO = 0.0;
  if constexpr (KC != ROW_PIVOT) {
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
      offP += code_offset(KC) * w.a[r * G::NG + rg];
      offO += code_offset(KC) * w.b[r * G::NG + rg];
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    accP[j] = -offP;
    accO[j] = -offO;
  }
#pragma unroll
  for (int r0 = 0; r0 < G::RPT; r0 += RB) {
    uint32_t wd[RB][NWD];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const uint8_t* row = rec + 2u * D + (uint32_t)((r0 + r) * G::NG + rg) * rb;
      chunk_words<KC == ROW_PIVOT ? 16 : KC, false, true>(row, cc, wd[r]);
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int i = (r0 + r) * G::NG + rg;
      if constexpr (KC == ROW_PIVOT)
        wrow_pivot(wd[r], w.a[i], w.b[i], accP, accO);
      else
        wrow_q<KC>(wd[r], w.a[i], w.b[i], accP, accO);
    }
  }
}

// The frozen pass of a mixed-width head: rows in the order of row_perm
// (rows of one width together), one row's words loaded ahead of its use.
template <int D>
__device__ __forceinline__ void wfrozen_mixed(const uint8_t* rec, const uint16_t* roff, const uint8_t* rcode,
                                              const uint8_t* rperm, uint32_t bytes, const WWork& w, int rg, int cc,
                                              double (&accP)[16], double (&accO)[16]) {
  using G = PGeo<D>;
  double offP = 0.0, offO = 0.0;
#pragma unroll 1
  for (int r = 0; r < G::RPT; ++r) {
    const int i = rperm[r * G::NG + rg] & (D - 1);
    const int code = rcode[i];
    if (code != ROW_PIVOT) {
      offP += code_offset(code) * w.a[i];
      offO += code_offset(code) * w.b[i];
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    accP[j] = -offP;
    accO[j] = -offO;
  }
  uint32_t nxt[8];
  int inext = rperm[rg] & (D - 1);
  int cnext = rcode[inext];
  wload_words(rec + min((uint32_t)roff[inext], bytes), cnext, cc, nxt);
#pragma unroll 1
  for (int r = 0; r < G::RPT; ++r) {
    uint32_t cur[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) cur[x] = nxt[x];
    const int i = inext, code = cnext;
    if (r + 1 < G::RPT) {
      inext = rperm[(r + 1) * G::NG + rg] & (D - 1);
      cnext = rcode[inext];
      wload_words(rec + min((uint32_t)roff[inext], bytes), cnext, cc, nxt);
    }
    const double ai = w.a[i];
    const double bi = w.b[i];
    switch (code) {
      case 8: wrow_q<8>(cur, ai, bi, accP, accO); break;
      case 6: wrow_q<6>(cur, ai, bi, accP, accO); break;
      case 4: wrow_q<4>(cur, ai, bi, accP, accO); break;
      case 2: wrow_q<2>(cur, ai, bi, accP, accO); break;
      default: wrow_pivot(cur, ai, bi, accP, accO); break;
    }
  }
}

// One tile. Returns status bits.
template <int D, int KC>
__device__ __forceinline__ uint32_t wtile(const WindowArgs& a, const WLay& L, uint8_t* stg, const WHdr* hd,
                                          const WWork& w, int rg, int cc) {
  using G = PGeo<D>;
  constexpr int NC = WGeo<D>::NC;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const bool kda = a.gate_kind != 0;
  const int W = a.W;
  const int n = hd->n;
  const int tile = hd->tile;
  const int h = tile % a.h_v;
  uint8_t* rec = hd->rec;
  const float* sq = reinterpret_cast<const float*>(stg + L.q);
  const float* sk = reinterpret_cast<const float*>(stg + L.k);
  const float* sv = reinterpret_cast<const float*>(stg + L.v);
  const float* sg = reinterpret_cast<const float*>(stg + L.g);
  const float* scol = reinterpret_cast<const float*>(stg + L.col);
  const float* sicol = reinterpret_cast<const float*>(stg + L.icol);
  const uint16_t* roff = reinterpret_cast<const uint16_t*>(stg + L.roff);
  const uint8_t* rcode = stg + L.rcode;
  const uint8_t* rperm = stg + L.rperm;
  const float* kb = reinterpret_cast<const float*>(stg + L.kb);
  float* ub = reinterpret_cast<float*>(stg + L.ub);  // turned into w rows at a window's end
  const float* gb = reinterpret_cast<const float*>(stg + L.gb);
  uint32_t st = 0;

  // ---- per key row i = tid: decays, E k products, a_i, b_i
  {
    const int i = tid;
    double acc = (double)(kda ? sg[i] : hd->g);  // prod over sigma = s .. n, from s = n down
#pragma unroll 1
    for (int s = n; s >= 1; --s) {
      w.ek[(s - 1) * D + i] = __dmul_rn(acc, (double)kb[(s - 1) * D + i]);
      acc = __dmul_rn(acc, (double)gb[kda ? (s - 1) * D + i : s - 1]);
    }
    const int code = KC ? KC : rcode[i];
    const float M = code == ROW_PIVOT ? 1.0f : __half2float(reinterpret_cast<const __half*>(rec)[i]);
    const double DM = __dmul_rn(acc, (double)M);
    const double ki = (double)sk[i], qi = (double)sq[i];
    w.a[i] = __dmul_rn(DM, ki);
    w.b[i] = __dmul_rn(DM, qi);
    w.kd[i] = ki;
    w.qd[i] = qi;
    w.d0[i] = acc;
    w.m[i] = M;
  }
  consumer_sync(NC);  // a, b, E k complete

  // ---- alpha_tau, gamma_tau (tau < n) and k.q (tau = n), one warp per tau
#pragma unroll 1
  for (int tau = warp; tau <= n; tau += G::NW) {
    double sa = 0.0, sgm = 0.0;
#pragma unroll
    for (int x = lane; x < D; x += 32) {
      const double kx = w.kd[x];
      const double e = tau < n ? w.ek[tau * D + x] : kx;
      sa = fma(e, kx, sa);
      sgm = fma(e, w.qd[x], sgm);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      sgm += __shfl_xor_sync(0xffffffffu, sgm, o);
    }
    if (lane == 0) {
      w.ag[tau] = sa;
      w.ag[W + tau] = sgm;
    }
  }

  // ---- frozen pass: column sums of the codes against a and b (fp64)
  {
    double accP[16], accO[16];
    if constexpr (KC != 0)
      wfrozen_uniform<D, KC>(rec, w, rg, cc, accP, accO);
    else
      wfrozen_mixed<D>(rec, roff, rcode, rperm, hd->bytes, w, rg, cc, accP, accO);
    wdeposit<D>(w.redp, warp, lane, cc, accP);
    wdeposit<D>(w.redo, warp, lane, cc, accO);
  }
  consumer_sync(NC);  // partials, alpha, gamma complete

  // ---- per column j = tid: p, u, o; append token n to the window
  {
    const int j = tid;
    const double Pt = wtotal<D>(w.redp, j);
    const double Ot = wtotal<D>(w.redo, j);
    const double cj = (double)scol[j];
    double p = __dmul_rn(cj, Pt);
    double oo = __dmul_rn(cj, Ot);
#pragma unroll 1
    for (int tau = 0; tau < n; ++tau) {
      const double u = (double)ub[tau * D + j];
      p = fma(w.ag[tau], u, p);
      oo = fma(w.ag[W + tau], u, oo);
    }
    const float un = __double2float_rn(__dmul_rn((double)hd->beta, __dsub_rn((double)sv[j], p)));
    oo = fma(w.ag[W + n], (double)un, oo);
    const float oj = __double2float_rn(oo);
    if (oj != oj) st |= ST_NAN;
    a.o[(size_t)tile * D + j] = oj;
    float* wk = reinterpret_cast<float*>(hd->wrec + 16);
    float* wu = wk + (size_t)W * D;
    float* wg = wu + (size_t)W * D;
    wk[n * D + j] = sk[j];
    wu[n * D + j] = un;
    if (kda)
      wg[n * D + j] = sg[j];
    else if (j == 0)
      wg[n] = hd->g;
    if (n + 1 < W) {
      if (j == 0) *reinterpret_cast<int32_t*>(hd->wrec) = n + 1;
      return st;
    }
    w.un[j] = __fmul_rn(un, sicol[j]);  // the current token's w
  }

  // ---- end of the window: T = V a + sum_tau e_tau w_tau in fp32, requantized
  // in place (the record's column-normalised units; see the oracle's
  // definition: t = fmaf(e, w, t) over the tokens in order, T = fmaf(V, a, t))
  consumer_sync(NC);  // w of the current token is in
  float* e = reinterpret_cast<float*>(stg + L.kb);  // [tau][row] over the buffered keys (used up)
  {
    const int i = tid;
    for (int tau = 0; tau < n; ++tau) e[tau * D + i] = __double2float_rn(w.ek[tau * D + i]);
    w.ecur[i] = sk[i];
    w.af[i] = __double2float_rn(__dmul_rn(w.d0[i], (double)w.m[i]));
    // as column j = i: the buffered u rows become w rows, each 16-column
    // chunk stored rotated (wswz) so that the lanes of a row group read
    // their chunks from different banks; the 16 columns of a chunk belong
    // to 16 lanes of one warp, which read before any of them writes
    const float icj = sicol[i];
    const int si = wswz(i);
    for (int tau = 0; tau < n; ++tau) {
      const float x = __fmul_rn(ub[tau * D + i], icj);
      __syncwarp();
      ub[tau * D + si] = x;
      __syncwarp();
    }
    const float xc = w.un[i];
    __syncwarp();
    w.un[si] = xc;
  }
  consumer_sync(NC);  // e, a, w complete
  const float* phi = a.t.phi + (size_t)h * D;
  constexpr bool DIRECT = KC == ROW_PIVOT;
#pragma unroll 1
  for (int grp = 0; grp < G::RPT / G::QS; ++grp) {
    int rows[G::QS];
#pragma unroll
    for (int u = 0; u < G::QS; ++u) {
      const int s = (grp * G::QS + u) * G::NG + rg;
      rows[u] = KC ? s : (rperm[s] & (D - 1));
    }
    float2 T[G::QS][8];
#pragma unroll
    for (int u = 0; u < G::QS; ++u)
#pragma unroll
      for (int p = 0; p < 8; ++p) T[u][p] = make_float2(0.0f, 0.0f);
    // t += e_tau (x) w_tau for the buffered tokens, then the current one
    auto add_token = [&](const float* wrow, const float* erow) {
      float2 wv[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 x = *reinterpret_cast<const float4*>(wrow + 16 * cc + 4 * ((p + (cc >> 1)) & 3));
        wv[2 * p] = make_float2(x.x, x.y);
        wv[2 * p + 1] = make_float2(x.z, x.w);
      }
#pragma unroll
      for (int u = 0; u < G::QS; ++u) {
        const float2 ev = f2(erow[rows[u]]);
#pragma unroll
        for (int p = 0; p < 8; ++p) T[u][p] = __ffma2_rn(ev, wv[p], T[u][p]);
      }
    };
#pragma unroll 2
    for (int tau = 0; tau < n; ++tau) add_token(ub + tau * D, e + tau * D);
    add_token(w.un, w.ecur);
#pragma unroll
    for (int u = 0; u < G::QS; ++u) {
      const int i = rows[u];
      float2 V[8];
      if constexpr (KC != 0) {
        constexpr uint32_t rb = KC == ROW_PIVOT ? 2u * D : (uint32_t)(D * KC / 8);
        row_values<KC == ROW_PIVOT ? 16 : KC, false, true>(rec + 2u * D + (uint32_t)i * rb, cc, V);
      } else {
        const uint8_t* row = rec + min((uint32_t)roff[i], hd->bytes);
        switch (rcode[i]) {
          case 8: row_values<8, false, false>(row, cc, V); break;
          case 6: row_values<6, false, false>(row, cc, V); break;
          case 4: row_values<4, false, false>(row, cc, V); break;
          case 2: row_values<2, false, false>(row, cc, V); break;
          default: row_values<16, false, false>(row, cc, V); break;
        }
      }
      const float2 av = f2(w.af[i]);
#pragma unroll
      for (int p = 0; p < 8; ++p) T[u][p] = __ffma2_rn(V[p], av, T[u][p]);
    }
    st |= prequant<D, KC, DIRECT>(rec, roff, rcode, rperm, phi, hd->bytes, grp, rg, cc, T);
  }
  if (tid == 0) *reinterpret_cast<int32_t*>(hd->wrec) = 0;
  return st;
}

template <int D>
__global__ void __launch_bounds__(WGeo<D>::NT, 3) k_window_step(const WindowArgs a) {
  using G = PGeo<D>;
  constexpr int NC = WGeo<D>::NC;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[2];
  __shared__ __align__(8) uint64_t empty[2];
  __shared__ uint32_t st_sh;
  __shared__ int abort_sh;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int gd = a.gate_kind != 0 ? D : 1;
  const WLay L = window_layout(D, a.W, gd);

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
    st_sh = 0;
    abort_sh = 0;
  }
  __syncthreads();

  if (warp == G::NW) {
    // ---------------- producer (lane 0)
    if (lane == 0) {
      const int n_tiles = a.B * a.h_v;
      WScal cur = wscal(a, blockIdx.x);
      WScal nxt = wscal(a, blockIdx.x + gridDim.x);
      int ncur = wcount(a, cur);
      int last_it[2] = {-1, -1};
      for (int it = 0;; ++it) {
        const int s = it & 1;
        uint8_t* stg = smem + (size_t)s * L.stage;
        // loads for the tiles after this one: issued now, used later
        const int nnxt = wcount(a, nxt);
        const WScal nn = wscal(a, blockIdx.x + (it + 2) * gridDim.x);
        if (it >= 2 && !wait_suspend(&empty[s], (uint32_t)((it >> 1) - 1) & 1u, a.wait_ns)) break;
        if (cur.m >= n_tiles) {
          reinterpret_cast<WHdr*>(stg)->tile = -1;
          mbar_arrive(&full[s]);
          // the stage's earlier copies were consumed (its empty barrier
          // said so), and this phase carries none
          last_it[s] = -1;
          break;
        }
        wissue<D>(a, L, stg, &full[s], cur, ncur);
        last_it[s] = it;
        cur = nxt;
        nxt = nn;
        ncur = nnxt;
      }
      // every bulk copy issued has landed before the CTA can exit (the phase
      // waited for is the stage's last one)
      for (int s = 0; s < 2; ++s)
        if (last_it[s] >= 0) (void)mbar_wait_bounded(&full[s], (uint32_t)(last_it[s] >> 1) & 1u, a.wait_ns);
    }
  } else {
    // ---------------- consumers
    const int cc = lane % G::LPR;
    const int rg = warp * G::RPW + lane / G::LPR;
    WWork w;
    w.redp = reinterpret_cast<double*>(smem + L.redp);
    w.redo = reinterpret_cast<double*>(smem + L.redo);
    w.ek = reinterpret_cast<double*>(smem + L.ek);
    w.a = reinterpret_cast<double*>(smem + L.a);
    w.b = reinterpret_cast<double*>(smem + L.b);
    w.kd = reinterpret_cast<double*>(smem + L.kd);
    w.qd = reinterpret_cast<double*>(smem + L.qd);
    w.d0 = reinterpret_cast<double*>(smem + L.d0);
    w.m = reinterpret_cast<float*>(smem + L.m);
    w.un = reinterpret_cast<float*>(smem + L.un);
    w.af = reinterpret_cast<float*>(smem + L.af);
    w.ecur = reinterpret_cast<float*>(smem + L.ecur);
    w.ag = reinterpret_cast<double*>(smem + L.ag);
    uint32_t st = 0;
    for (int it = 0;; ++it) {
      const int s = it & 1;
      uint8_t* stg = smem + (size_t)s * L.stage;
      const WHdr* hd = reinterpret_cast<const WHdr*>(stg);
      // a thread that gives up records the iteration, so that every consumer
      // takes the same decision after the barrier
      if (!wait_suspend(&full[s], (uint32_t)(it >> 1) & 1u, a.wait_ns)) abort_sh = it + 1;
      consumer_sync(NC);  // stage s is in for every consumer, or someone gave up
      if (tid == 0 && it > 0) mbar_arrive(&empty[s ^ 1]);  // the previous tile is done
      if (*reinterpret_cast<volatile int*>(&abort_sh) == it + 1) {
        st |= ST_TIMEOUT;
        break;
      }
      const int tile = hd->tile;
      if (tile < 0) break;
      if (hd->valid != 1) {
        a.o[(size_t)tile * D + tid] = 0.0f;
        st |= hd->valid == 0 ? ST_SLOT : ST_WINDOW;
        continue;
      }
      switch (hd->kind) {
        case 8: st |= wtile<D, 8>(a, L, stg, hd, w, rg, cc); break;
        case 6: st |= wtile<D, 6>(a, L, stg, hd, w, rg, cc); break;
        case 4: st |= wtile<D, 4>(a, L, stg, hd, w, rg, cc); break;
        case 2: st |= wtile<D, 2>(a, L, stg, hd, w, rg, cc); break;
        case ROW_PIVOT: st |= wtile<D, ROW_PIVOT>(a, L, stg, hd, w, rg, cc); break;
        default: st |= wtile<D, 0>(a, L, stg, hd, w, rg, cc); break;
      }
    }
    if (st) atomicOr(&st_sh, st);
  }
  __syncthreads();
  if (tid == 0 && st_sh) atomicOr(a.t.status, st_sh);
}

}  // namespace sqk
