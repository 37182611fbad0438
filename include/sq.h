/*
 * sq.h -- C ABI of the quantized recurrent-state decode step for gated
 * delta-rule linear attention (GDN: one gate per head; KDA: one gate per key
 * channel), B200 (sm_100a).
 *
 * The method (STEPQuant): every request keeps, per value head, a d x d state
 * S (row i = key channel, column j = value channel) that a decode step
 * updates with the gated delta rule
 *     S <- diag(g) S ;  u = beta (v - S^T k) ;  S <- S + k u^T ;  o = S^T q
 * ("STEPQuant review (e-cogni)", section "Contexto"; "STEPQuant talk
 * announcement (qingkeai)", opening section). Between steps the state lives
 * in a compressed form, S_ij ~= r_i c_j q_ij, with a row scale per key row
 * taken from the row's current magnitude and its calibrated row-impact
 * factor, a calibrated column scale per value column, and low-bit codes
 * whose width is set per unit (a head for GDN, a key row for KDA); a few
 * units are kept as FP16 pivots ("STEPQuant review (e-cogni)", section
 * "O que os autores propõem"; "STEPQuant: estados recurrentes a 6 bit"
 * (gpt-diffusion), section "Las dos ideas: cuándo y dónde importa el
 * error"). Each step reads that state once, updates it in FP32, and
 * requantizes it in place ("STEPQuant: estados recurrentes a 6 bit",
 * "Las dos ideas", fused kernels on packed states).
 *
 * Conventions for every call:
 *  - Pointers named "device" are CUDA device pointers on the device that was
 *    current when the handle was created; they must be 16-byte aligned and
 *    the arrays C-contiguous. Pointers named "host" are host memory.
 *  - Every call that takes a stream is asynchronous on that stream
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream),
 *    except sq_get_status, which synchronizes it.
 *  - Invalid arguments are rejected on the host with SQ_ERR_INVALID_ARG and
 *    nothing is launched; sq_last_error() then returns a message.
 *  - Bad data found on the device (NaN, fp16 overflow, a slot id out of
 *    range) never traps: the kernel writes defined values and ORs a bit into
 *    the handle's device status word (SQ_STATUS_*), read by sq_get_status.
 *  - There is no CPU fallback: without a usable CUDA device every call that
 *    launches work returns SQ_ERR_CUDA.
 *  - Calls on one handle from different host threads must be serialized by
 *    the caller. Two steps in flight on the same pool slots race. Steps of
 *    one handle must also not run at the same time on the device (e.g. on
 *    two unordered streams): they share the handle's work counter, which
 *    each step leaves at zero when it ends.
 *
 * Storage format (SQ_FMT_PACKED). The pool is caller-owned device memory of
 * sq_state_bytes().pool_bytes bytes. Slot s starts at s * slot_bytes; in it
 * the value heads follow each other (sq_head_layout gives each head's
 * offset and record size). A head record is
 *     [d row scales r_i, fp16 LE][row 0][row 1] ... [row d-1][zero pad to 16 B]
 * A pivot row is d fp16 values of the column-normalised state T = S / c
 * (its scale slot holds fp16 1.0). A quantized row of width b in {2,4,6,8}
 * is a little-endian bit stream of d fields of b bits: field j holds
 * q_ij + 2^(b-1) (offset binary), q_ij in [-(2^(b-1)-1), 2^(b-1)-1].
 * SQ_FMT_FP32 pools are plain fp32 S [n_slots][h_v][d][d].
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,  /* rejected on the host; nothing launched */
  SQ_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. d not in {32, 64, 128}) */
  SQ_ERR_CUDA = 3,         /* a CUDA runtime call failed; see sq_last_error() */
  SQ_ERR_OOM = 4           /* device allocation of the handle's tables failed */
} sq_status;

typedef enum { SQ_FMT_FP32 = 0, SQ_FMT_PACKED = 1 } sq_format;
typedef enum { SQ_GATE_HEAD = 0 /* GDN */, SQ_GATE_KEY_CHANNEL = 1 /* KDA */ } sq_gate_kind;

/* Bits of the device status word. */
#define SQ_STATUS_NAN 1u        /* a NaN reached the updated state or o */
#define SQ_STATUS_SATURATED 2u  /* a row scale or pivot value saturated at +-65504 */
#define SQ_STATUS_BAD_SLOT 4u   /* a slot id outside [0, n_slots) was skipped (o = 0) */
#define SQ_STATUS_TIMEOUT 8u    /* a bounded device wait gave up (should never happen) */
#define SQ_STATUS_WINDOW 16u    /* sq_window_step: a window record's count was outside [0, W);
                                   the tile was skipped (o = 0, nothing written) */

/* Shape of one layer's state pool. d_k == d_v == d, d in {32, 64, 128};
 * h_v % h_k == 0 (value head h reads key head h / (h_v / h_k)). */
typedef struct {
  int32_t n_slots;   /* requests the pool can hold */
  int32_t h_v;       /* value heads (states per request) */
  int32_t h_k;       /* key heads */
  int32_t d_k;
  int32_t d_v;
  int32_t fmt;       /* sq_format */
  int32_t gate;      /* sq_gate_kind */
} sq_state_desc;

/* Calibration tables, host memory, copied by sq_state_alloc (the caller
 * keeps ownership). Units are heads (GATE_HEAD) or key rows (GATE_KEY_CHANNEL).
 * Ignored (may be NULL) for SQ_FMT_FP32. */
typedef struct {
  const int8_t* unit_bits;    /* [h_v] or [h_v*d_k]; 2, 4, 6 or 8 */
  const uint8_t* pivot_mask;  /* same shape; nonzero = FP16 pivot unit (overrides unit_bits) */
  const float* col_scale;     /* [h_v*d_v] c_j, finite and > 0 */
  const float* row_impact;    /* [h_v*d_k] phi_i, finite and > 0; used as the clip ratio min(phi_i, 1) */
} sq_calib;

typedef struct sq_handle sq_handle;

typedef struct {
  uint64_t pool_bytes;             /* n_slots * slot_bytes */
  uint64_t slot_bytes;             /* one request's state, all heads */
  uint64_t state_bytes_per_step;   /* per request: slot read + slot written by one step */
  uint64_t act_bytes_per_step;     /* per request: q, k, v, beta, g read and o written */
  double bits_per_value;           /* 8 * slot_bytes / (h_v * d_k * d_v) */
  uint64_t max_record_bytes;       /* largest head record */
} sq_bytes_report;

/* Plumbing (no passage of the method's pages: handle, layout and error
 * reporting around the steps). Create a handle: validate the description
 * and calibration, build the
 * record layout and upload the per-head tables (ic_j = 1/c_j included) to
 * the current device with cudaMalloc + cudaMemcpyAsync on `stream`. The
 * state pool itself is NOT allocated: the caller allocates pool_bytes
 * (returned in *pool_bytes) of device memory. Returns SQ_ERR_INVALID_ARG for
 * bad shapes or tables, SQ_ERR_UNSUPPORTED for d not in {32, 64, 128},
 * SQ_ERR_OOM if the tables cannot be allocated. */
sq_status sq_state_alloc(const sq_state_desc* desc, const sq_calib* calib, void* stream,
                         sq_handle** out, size_t* pool_bytes);

/* Plumbing (no passage). Release the handle's device tables (synchronizes
 * the device first). NULL is a no-op. */
sq_status sq_state_free(sq_handle* h);

/* Quantize B fp32 states into pool slots ("STEPQuant review (e-cogni)",
 * "O que os autores propõem", dual-axis fitting: T = S / c, row scales from
 * the current row magnitude times phi, codes rounded to nearest even).
 *   S        device fp32 [B, h_v, d, d], S-space (row = key channel)
 *   slot_ids device int32 [B], or NULL for slots 0..B-1
 * B == 0 is a no-op. FP32 pools: a plain copy. */
sq_status sq_quantize_state(sq_handle* h, void* pool, const float* S, const int32_t* slot_ids,
                            int32_t B, void* stream);

/* One decode step for B requests, in place on the pool ("STEPQuant review
 * (e-cogni)", "Contexto": gated delta rule; talk announcement, "STEPQuant
 * 核心设计": row scales from magnitude and impact, column scales; gpt-diffusion
 * page, "Las dos ideas": fused kernels on packed states):
 *   q, k     device fp32 [B, h_k, d]
 *   v        device fp32 [B, h_v, d]
 *   beta     device fp32 [B, h_v]
 *   g        device fp32 [B, h_v] (GATE_HEAD) or [B, h_v, d] (GATE_KEY_CHANNEL)
 *   o        device fp32 [B, h_v, d], written: o = S'^T q from the updated
 *            state before requantization
 *   slot_ids device int32 [B] (distinct), or NULL for slots 0..B-1
 * Reads and writes each touched state record exactly once. */
sq_status sq_decode_step(sq_handle* h, void* pool, const float* q, const float* k, const float* v,
                         const float* beta, const float* g, float* o, const int32_t* slot_ids,
                         int32_t B, void* stream);

/* The same decode step with the activations in HOST memory, for a caller
 * that keeps them there (the method's paper has no counterpart; this is the
 * serving loop's host-to-device boundary). q, k, v, beta, g and slot_ids
 * (or NULL) are host arrays of the shapes of sq_decode_step; o is a host
 * array [B, h_v, d] written by the step.
 *   - The inputs are copied on an internal stream into one of two device
 *     staging sets owned by the handle (allocated at the first call and
 *     whenever B grows, which synchronizes the device); the copies of a call
 *     wait only for the step that last used the same set, so they overlap
 *     the step of the previous call. The step itself runs on `stream` after
 *     its copies. Page-locked inputs make the copies asynchronous; pageable
 *     ones are accepted but the copies then block the host.
 *   - o in mapped page-locked memory (cudaHostAlloc, cudaMallocHost, or
 *     registered memory on a system with unified addressing) is written by
 *     the kernel directly over the bus; any other o is staged and copied
 *     back on `stream`.
 *   - The host inputs must stay unchanged, and o must not be read, until
 *     `stream` has passed this call (e.g. cudaStreamSynchronize).
 * Every step of one handle, device- or host-buffer, must run on one stream
 * (or streams the caller orders), as for sq_decode_step. */
sq_status sq_decode_step_host(sq_handle* h, void* pool, const float* q, const float* k, const float* v,
                              const float* beta, const float* g, float* o, const int32_t* slot_ids, int32_t B,
                              void* stream);

/* Per-window variant of the decode step ("线性注意力每生成一个token都要搬状态，
 * LeapQuant把它压到8位还不掉点" (wink.run), per-window quantization, the first
 * of LeapQuant's three techniques): the packed state of a tile is frozen for
 * a window of W tokens; every token's key k, update vector u and gate go to
 * a high-precision buffer, the outputs come from the frozen state and the
 * buffer together, and the state is requantized once when the window is
 * full. The page gives no formula; the step computes, for a tile with n
 * buffered tokens (this token is token n, its gate G_n; products of gates
 * E_tau,i = G_{tau+1},i ... G_n,i, E_-1 over all n + 1 tokens):
 *     S_ij = E_-1,i S0_ij + sum_{tau<n} E_tau,i k_tau,i u_tau,j   (S0 the frozen state)
 *     u_j  = fp32(beta (v_j - sum_i S_ij k_i))
 *     o_j  = fp32(sum_i (S_ij + k_i u_j) q_i)
 * in fp64 (u and o rounded once), and appends (k, u, G_n) as row n of the
 * buffer. At n + 1 = W it forms the state in the record's column-normalised
 * units in fp32, the way sq_decode_step forms its updated state:
 *     T_ij = fmaf(V_ij, a_i, t_ij),  t_ij = fmaf(e_tau,i, w_tau,j, t_ij) over
 *     tau = 0 .. W-1 from t = 0,  a_i = fp32(E_-1,i M_i) (M_i the row scale,
 *     1 for a pivot row), e_tau,i = fp32(E_tau,i k_tau,i) (E = 1 for the last
 *     token), w_tau,j = fp32(u_tau,j fp32(1 / c_j)),
 * requantizes T in place with the rules of sq_decode_step and empties the
 * buffer. Inside a window the pool is only read.
 *   window_buf device, sq_window_buffer_bytes() bytes, caller-owned; record
 *            of (slot s, value head h) at (s h_v + h) record_bytes:
 *            [int32 count, 12 zero bytes][k: W x d fp32][u: W x d fp32]
 *            [gates: W x gd fp32, zero-padded to a multiple of 4 floats],
 *            gd = d (GATE_KEY_CHANNEL) or 1 (GATE_HEAD); row tau holds
 *            buffered token tau. A slot whose state is (re)written by
 *            sq_quantize_state or sq_prefill must have its records zeroed
 *            (count 0) before its next window step. While count > 0 the
 *            pool holds the state from before the buffered tokens.
 *   W        window length, 1 <= W <= 64 (W = 1 is per-token
 *            requantization, with fp64 instead of fp32 arithmetic); the
 *            same W for every call on one buffer.
 *   q .. o, slot_ids, B: as sq_decode_step (slot ids distinct).
 * A count outside [0, W) skips the tile (o = 0, SQ_STATUS_WINDOW). Returns
 * SQ_ERR_INVALID_ARG for an FP32 pool, W out of range, or a W whose
 * working set does not fit in shared memory. */
sq_status sq_window_step(sq_handle* h, void* pool, void* window_buf, int32_t W, const float* q, const float* k,
                         const float* v, const float* beta, const float* g, float* o, const int32_t* slot_ids,
                         int32_t B, void* stream);

/* Plumbing (no passage). Sizes of the window buffer of sq_window_step for
 * windows of W tokens: bytes of one (slot, head) record and of the whole
 * buffer (n_slots h_v records). Returns SQ_ERR_INVALID_ARG for W outside
 * [1, 64]. */
sq_status sq_window_buffer_bytes(const sq_handle* h, int32_t W, uint64_t* record_bytes, uint64_t* buffer_bytes);

/* Expand B pool slots to fp32 S [B, h_v, d, d] (device): S_ij = (q r) c_j for
 * quantized rows and h c_j for pivot rows. Skipped (bad) slots give 0. */
sq_status sq_dequantize_state(sq_handle* h, const void* pool, float* S_out, const int32_t* slot_ids,
                              int32_t B, void* stream);

/* Prefill handoff: run the gated delta rule over a whole prompt for B
 * requests and write the final state once into their pool slots, quantized
 * for SQ_FMT_PACKED ("STEPQuant review (e-cogni)", "Contexto": the state a
 * prompt leaves behind is what every decode step then updates; "O que os
 * autores propõem": it enters the cache in the dual-axis quantized form).
 * One launch; each (request, head) state stays on chip for the whole
 * prompt. Token t of request b applies exactly the FP32 decode step of
 * sq_decode_step on an SQ_FMT_FP32 pool (same arithmetic and summation
 * order), so the final fp32 state equals that of L such steps bit for bit;
 * the quantization is that of sq_quantize_state.
 *   S0       device fp32 [B, h_v, d, d] initial state, or NULL for zeros
 *   q, k     device fp32 [B, L, h_k, d]
 *   v        device fp32 [B, L, h_v, d]
 *   beta     device fp32 [B, L, h_v]
 *   g        device fp32 [B, L, h_v] (GATE_HEAD) or [B, L, h_v, d] (GATE_KEY_CHANNEL)
 *   o        device fp32 [B, L, h_v, d], written for t < lengths[b]: o_t = S_t^T q_t
 *   S_out    device fp32 [B, h_v, d, d] final state (unquantized), or NULL
 *   lengths  device int32 [B] prompt lengths (values outside [0, L] are
 *            clamped), or NULL for L; a length of 0 stores S0 (or zeros)
 *   slot_ids device int32 [B] (distinct), or NULL for slots 0..B-1; an
 *            out-of-range slot is skipped (SQ_STATUS_BAD_SLOT), o and S_out
 *            are still written
 * q, k, v, o, S0 and S_out 16-byte aligned; g too for GATE_KEY_CHANNEL.
 * B == 0 is a no-op; L == 0 stores S0 (or zeros). */
sq_status sq_prefill(sq_handle* h, void* pool, const float* S0, const float* q, const float* k, const float* v,
                     const float* beta, const float* g, float* o, float* S_out, const int32_t* lengths,
                     const int32_t* slot_ids, int32_t B, int32_t L, void* stream);

/* Byte accounting of the layout (host only, no device work); the per-step
 * figures are the algorithmic bytes of Table D3's accounting applied to
 * this layout ("STEPQuant: estados recurrentes a 6 bit" (gpt-diffusion),
 * section on what the "6-bit" and the "68,7%" mean). */
sq_status sq_state_bytes(const sq_handle* h, sq_bytes_report* out);

/* Plumbing (no passage). Offset within a slot and size of value head
 * `head`'s record (host only). */
sq_status sq_head_layout(const sq_handle* h, int32_t head, uint64_t* offset, uint64_t* record_bytes);

/* Plumbing (no passage). Synchronize `stream`, return the device status
 * bits accumulated since the last clear, and clear them if `clear` is
 * nonzero. */
sq_status sq_get_status(sq_handle* h, void* stream, uint32_t* bits, int32_t clear);

/* Number of columns whose S^T k the packed decode steps of this handle have
 * summed with the exact fixed-point accumulator since the last clear. The
 * step defines S^T k as the exact value of the sum rounded once to fp32
 * (the reading of the quantize-after-every-update loop in "STEPQuant review
 * (e-cogni)", section "Contexto": the state feeds its own rounding back
 * every step, so the rounding must not depend on summation order); the
 * kernel sums in fp64, rounds when a rigorous error bound shows the fp64
 * total rounds like the exact value, and sums the column exactly otherwise.
 * This counts the latter (a diagnostic; rare on real data). Synchronizes
 * `stream`; clears the count if `clear` is nonzero. */
sq_status sq_get_exact_count(sq_handle* h, void* stream, uint32_t* count, int32_t clear);

/* Plumbing (no passage). Limit, in nanoseconds, of every bounded wait inside
 * this handle's step kernels (default 2 s; at least 1000). A wait that runs
 * out abandons its tile before anything of it is written and sets
 * SQ_STATUS_TIMEOUT. */
sq_status sq_set_wait_limit(sq_handle* h, uint64_t ns);

/* Testing only (no passage). From the next packed decode step on, the
 * shared-memory stage that receives tile (request 0, head 0) expects
 * `extra_bytes` (at most 65536) more bytes than are loaded into it, so the
 * wait of the CTA that took that tile runs out after the wait limit: the
 * step sets SQ_STATUS_TIMEOUT, that CTA leaves without writing any part of
 * the tiles it had taken, and the other CTAs finish the rest. 0 restores
 * normal operation. Every copy issued still lands; nothing is left in flight. */
sq_status sq_test_stall_stages(sq_handle* h, uint32_t extra_bytes);

/* Plumbing (no passage). Launch configuration of this handle's decode step
 * kernel (host only): grid size (persistent CTAs), threads per CTA, CTAs
 * resident per SM, shared-memory stages per CTA and dynamic shared-memory
 * bytes per CTA. Any pointer may be NULL. */
sq_status sq_launch_plan(const sq_handle* h, int32_t* grid, int32_t* threads, int32_t* ctas_per_sm,
                         int32_t* stages, int32_t* smem_bytes);

/* Plumbing (no passage). Number of kernel launches this handle has issued
 * (host-side counter). */
uint64_t sq_launch_count(const sq_handle* h);

/* Decode step that allocates nothing. The method's paper has no
 * counterpart; this entry point exists for callers that cannot allocate
 * device memory: a serving engine whose allocator has already reserved the
 * GPU's memory for its own pools (a cudaMalloc behind its back would fail
 * or fragment it), or a latency-critical caller that cannot afford the
 * device synchronization cudaMalloc may imply. It does the same step as
 * sq_decode_step on a packed pool laid out exactly as sq_state_alloc lays
 * it out for the same `desc` and `calib`, but without a handle:
 *   - the per-head tables (record and row offsets, widths, c, 1/c, phi)
 *     are rebuilt on the host from `calib` at every call and copied into a
 *     fixed 160 KiB array in device memory that this library declares at
 *     file scope (every GPU that loads the library holds it until the
 *     process exits); nothing is allocated on the device or the host heap;
 *   - limits: packed pools only, h_v <= SQ_NOALLOC_MAX_HEADS, and the tables
 *     must fit the array (h_v * d <= 8192 always does); larger shapes are
 *     rejected with SQ_ERR_UNSUPPORTED and a message;
 *   - the first call on a device looks up the array's device address and
 *     sets the kernels' shared-memory limit for that device;
 *   - the tables reach the array by an asynchronous copy from a host
 *     buffer that every call overwrites, so the call must not be made while
 *     `stream` is being captured into a CUDA graph: it then returns
 *     SQ_ERR_UNSUPPORTED and launches nothing;
 *   - every call shares the one array, which keeps the last call's tables:
 *     calls on the same device serialize on the host, but calls whose GPU
 *     work overlaps (different streams, or a later call before the earlier
 *     one's kernel ran) race on the array;
 *   - status: device pointer to a uint32 the kernel ORs SQ_STATUS_* bits
 *     into (the caller clears it), or NULL to discard the bits.
 * Other arguments as in sq_decode_step. */
#define SQ_NOALLOC_MAX_HEADS 64
sq_status sq_decode_step_noalloc(const sq_state_desc* desc, const sq_calib* calib, void* pool, const float* q,
                                 const float* k, const float* v, const float* beta, const float* g, float* o,
                                 const int32_t* slot_ids, int32_t B, uint32_t* status, void* stream);

/* Plumbing (no passage). Message for the last non-OK return on this host
 * thread ("" if none). */
const char* sq_last_error(void);

/* Plumbing (no passage). Library version string. */
const char* sq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SQ_H */
