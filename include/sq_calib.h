/*
 * sq_calib.h -- C ABI of the offline calibration that produces the decode
 * step's tables (sq_calib in sq.h) from traces, B200 (sm_100a).
 *
 * The method's calibration ("STEPQuant talk announcement (qingkeai)",
 * section "STEPQuant 核心设计"; "STEPQuant review (e-cogni)", sections
 * "O que os autores propõem" and "Como funciona"): a unit's precision is set
 * by its quantization error together with how long its memory lives (the
 * gate's retention), under a fixed bit budget, and the riskiest units stay
 * FP16 as sparse pivots; row scales carry a row-impact factor measured on
 * the readout; column scales are fitted with more weight on high-impact
 * rows; both axes are square-root smoothed and normalised to a geometric
 * mean of one. The pages state these ideas without formulas; this library
 * implements the following reading of them (M2, E[q^2] and the mean gates
 * are running fp64 sums over the trace, in trace order):
 *
 *   M2_ij    = sum_t S_t,ij^2                       per value head
 *   phi_i    = sqrt(max(E[q_i^2], 1e-6 max_k E[q_k^2])) / geomean
 *   rho_j    = sqrt(sum_i phi_i^2 M2_ij / (n sum_i phi_i^2))
 *   c_j      = sqrt(max(rho_j, 1e-12 max_k rho_k)) / geomean
 *   sigma2_u = mean over the unit's entries and samples of (S / c)^2
 *   w_u      = 1 / (1 - min(mean gate_u, 1 - 1e-6))  (expected lifetime)
 *   D_u(b)   = w_u sigma2_u 4^-b
 *   pivots   = the round-half-up(pivot_frac N) units of largest D_u(b_max)
 *              (ties: lower unit index), counted at b_max in the budget;
 *   widths   = all other units start at the narrowest allowed width; while
 *              a raise to the next allowed width fits the remaining budget
 *              nominal_bits * N, the raise with the largest drop of D is
 *              taken (ties: lower unit index).
 * A head whose queries (states) are all zero gets phi = 1 (c = 1).
 * Units are value heads (SQ_GATE_HEAD, N = h_v) or key rows
 * (SQ_GATE_KEY_CHANNEL, N = h_v * d).
 *
 * Conventions as in sq.h: device pointers 16-byte aligned and C-contiguous,
 * calls asynchronous on `stream` except sq_calib_finish, bad arguments
 * rejected on the host with SQ_ERR_INVALID_ARG before any launch,
 * sq_last_error() holds the message. Calls on one trace from different host
 * threads must be serialized by the caller; the trace's accumulators are
 * updated in stream order, so all calls on one trace must use one stream (or
 * streams the caller orders).
 */
#ifndef SQ_CALIB_H
#define SQ_CALIB_H

#include <stdint.h>

#include "sq.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sq_calib_trace sq_calib_trace;

/* The bit budget: allowed widths as a bit mask (bit b set = width b allowed,
 * b in {2, 4, 6, 8}, at least one), the nominal mean width per unit (between
 * the narrowest and the widest allowed width) and the fraction of units kept
 * as FP16 pivots (in [0, 1]). */
typedef struct {
  int32_t widths_mask;
  int32_t nominal_bits;
  double pivot_frac;
} sq_calib_budget;

/* Host output arrays of sq_calib_finish; the caller owns them. The first
 * four are exactly the tables sq_calib takes; the last two may be NULL. */
typedef struct {
  int8_t* unit_bits;    /* [N] width of each unit (pivots carry the widest) */
  uint8_t* pivot_mask;  /* [N] 1 = FP16 pivot unit */
  float* col_scale;     /* [h_v * d] c_j */
  float* row_impact;    /* [h_v * d] phi_i */
  double* unit_sigma2;  /* [N] sigma2_u, or NULL */
  double* unit_weight;  /* [N] w_u, or NULL */
} sq_calib_out;

/* Create an empty trace for the shape in `desc` (n_slots and fmt are
 * ignored; d_k == d_v == d in {32, 64, 128}, h_v % h_k == 0): allocates and
 * zeroes its fp64 accumulators on the current device, on `stream`.
 * SQ_ERR_OOM if the allocation fails. */
sq_status sq_calib_begin(const sq_state_desc* desc, void* stream, sq_calib_trace** out);

/* Add n state samples: S device fp32 [n, h_v, d, d] (row = key channel),
 * e.g. an SQ_FMT_FP32 pool of n slots. One HBM-bound kernel; n == 0 is a
 * no-op. */
sq_status sq_calib_add_states(sq_calib_trace* t, const float* S, int32_t n, void* stream);

/* Add n tokens: q device fp32 [n, h_k, d]; g device fp32 [n, h_v]
 * (SQ_GATE_HEAD) or [n, h_v, d] (SQ_GATE_KEY_CHANNEL). Either pointer may
 * be NULL to add only the other one (each keeps its own token count).
 * n == 0 is a no-op. */
sq_status sq_calib_add_tokens(sq_calib_trace* t, const float* q, const float* g, int32_t n, void* stream);

/* Compute the tables from everything added so far: one kernel (phi, c,
 * sigma2 per head), a copy to the host, the allocation on the host. Waits
 * for `stream`. SQ_ERR_INVALID_ARG if no state, query or gate was added, if
 * the budget is invalid, or if the trace held non-finite values (a phi or
 * c that is not finite and positive). The trace stays usable (more samples
 * may be added and finish called again). */
sq_status sq_calib_finish(sq_calib_trace* t, const sq_calib_budget* budget, const sq_calib_out* out,
                          void* stream);

/* The width allocation alone, on the host (no device work): the widths and
 * FP16 pivots sq_calib_finish chooses for N units with mean squares
 * sigma2[N] and lifetime weights weight[N] (host arrays, finite and >= 0)
 * under `budget` (rules in the header comment above). For callers that
 * compute the unit statistics themselves. unit_bits and pivot_mask are host
 * arrays of N entries. */
sq_status sq_calib_allocate(const double* sigma2, const double* weight, int64_t n, const sq_calib_budget* budget,
                            int8_t* unit_bits, uint8_t* pivot_mask);

/* Release the trace (synchronizes the device first). NULL is a no-op. */
sq_status sq_calib_free(sq_calib_trace* t);

#ifdef __cplusplus
}
#endif
#endif /* SQ_CALIB_H */
