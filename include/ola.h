/*
 * ola.h — C ABI of the beam-parallel Gated DeltaNet decode library (sm_100a).
 *
 * What the library computes
 * -------------------------
 * One GDN layer of R requests x H heads. Every request decodes B beams that all start from
 * one shared post-prefill state S_ctx (d_v x d_k per request and head). Decode step t of new
 * beam b continues parent beam p = parent_idx[r][b] of step t-1 ("Scientific Impact
 * Assessment: OneLA", §1 Core Contribution: hundreds of beams start from one prompt-derived
 * state and diverge through a few decode-time transitions; pruning, reordering and fan-out
 * are expressed by the ancestry index). The transition is the gated delta rule (Gated Delta
 * Networks, listed under "Builds on" on the OneLA listing):
 *
 *     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   alpha_t = exp(g_t)
 *     o_t = S_t q_t
 *
 * The default (replay) path never forms a per-beam state. Each beam appends a transition
 * record (w_t, k_t, alpha_t) with u_t = S_{t-1} k_t and w_t = beta_t (v_t - alpha_t u_t), so
 * that S_t = alpha_t S_{t-1} + w_t k_t^T, and S_{t-1} x is evaluated as
 *     (prod alpha) S_ctx x + sum_j (prod_{i>j} alpha_i) w_j (k_j . x)
 * over the records of the beam's chain ("Scientific Impact Assessment: OneLA", §1: append-only
 * records of O(d_v + d_k) per beam, projection replay through the key and query
 * contractions, one kernel reusing S_ctx across beams; the OneLA listing's Abstract: records
 * are never moved or copied when beams are updated). Two comparison paths implement the
 * practices the Abstract contrasts with: FullState keeps one d_v x d_k state per beam, and the
 * history-replay path (REPLAYSSM) keeps no state at all and rebuilds every beam's state from
 * S_ctx over its chain's raw tokens at every step.
 *
 * Conventions (every entry point)
 * -------------------------------
 * - Tensors are row-major, contiguous, on the current CUDA device unless a function says
 *   "host". Layouts are given in brackets, slowest index first.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Calls are
 *   stream-ordered and asynchronous unless stated; inputs are borrowed only until the work
 *   queued on `stream` has run; the library never keeps a caller pointer.
 * - Host-side validation failures return at once, with nothing launched and no state changed.
 * - Device-side errors (an out-of-range parent, a bounded wait that ran out) are sticky: the
 *   kernel clamps and carries on and records the first code in a device word. ola_get_error
 *   waits for the handle's queued work and returns it; from then on ola_step refuses to run
 *   (returns that code, launches nothing) until ola_reset clears it. Outputs of a step that
 *   recorded an error are unspecified.
 * - A handle is used by one host thread at a time.
 * - Pointers to q, k, v, out_o and S_ctx must be 16-byte aligned; g, beta, parent_idx
 *   4-byte aligned.
 */
#ifndef OLA_H_
#define OLA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OLA_OK = 0,
  OLA_ERR_INVALID_ARG = 1,   /* NULL / misaligned pointer, bad size, bad enum */
  OLA_ERR_UNSUPPORTED = 2,   /* geometry outside what this build supports, or not sm_100 */
  OLA_ERR_CAPACITY = 3,      /* ola_step after T_max steps (nothing launched) */
  OLA_ERR_BAD_PARENT = 4,    /* a parent index was out of range (device-detected, sticky) */
  OLA_ERR_OOM = 5,           /* device allocation failed */
  OLA_ERR_CUDA = 6,          /* a CUDA runtime call failed */
  OLA_ERR_TIMEOUT = 7,       /* a bounded device wait ran out (device-detected, sticky) */
  OLA_ERR_SCRATCH_LIMIT = 8  /* ola_decode_noalloc: problem larger than its fixed scratch */
} ola_status;

/* dtype of q, k, v (and of the prompt's k, v for ola_prefill) */
enum { OLA_F32 = 0, OLA_BF16 = 1 };
/* how beam states are represented:
 * REPLAY     = one shared state + append-only transition records (w, k, alpha) per beam,
 *              evaluated by projection replay (the method);
 * FULLSTATE  = one materialised d_v x d_k fp32 state per beam, ping-pong buffers (comparison);
 * REPLAYSSM  = no per-beam state kept: each step rebuilds every beam's state from the shared
 *              state by replaying the raw tokens (k, v, alpha, beta) on its chain, fp32
 *              (comparison). */
enum { OLA_PATH_REPLAY = 0, OLA_PATH_FULLSTATE = 1, OLA_PATH_REPLAYSSM = 2 };
/* how the contractions of the replay path are computed:
 * FP32 = CUDA-core fp32 FMA everywhere; TENSOR = tcgen05 tensor cores, bf16 operands with
 * S_ctx split into a bf16 high part and a bf16 remainder (two MMAs, fp32 accumulate in
 * tensor memory). With B <= 1024 and T_max <= 12 the replay accumulation over the ancestor
 * records also runs on tensor cores: the records' w rows are then kept as a bf16 high part and
 * a bf16 remainder (same bytes as fp32) and each product runs as three bf16 MMAs with fp32
 * accumulation; beyond those limits it runs in fp32 on CUDA cores. */
enum { OLA_MATH_FP32 = 0, OLA_MATH_TENSOR = 1 };

typedef struct {
  int32_t R;          /* requests, >= 1 */
  int32_t H;          /* heads, >= 1 */
  int32_t d_k;        /* key width: 16, 32, 64, 128 or 256 (TENSOR: 64, 128, 256) */
  int32_t d_v;        /* value width: 16, 32, 64, 128 or 256 (TENSOR: 64, 128, 256) */
  int32_t B;          /* beams per request, 1..4096 (TENSOR: T_max*R*H*B < 2^31) */
  int32_t T_max;      /* decode steps the handle can hold, 1..32 */
  int32_t in_dtype;   /* OLA_F32 or OLA_BF16 (TENSOR: OLA_BF16) */
  int32_t path;       /* OLA_PATH_REPLAY, OLA_PATH_FULLSTATE or OLA_PATH_REPLAYSSM */
  int32_t math;       /* OLA_MATH_FP32 or OLA_MATH_TENSOR (replay path only) */
} ola_geometry;

typedef struct ola_ctx* ola_handle;

/* Library version, (major << 16) | minor. Never fails, touches no device. */
int32_t ola_version(void);

/* Static message for a status code. Never fails, touches no device. */
const char* ola_strerror(ola_status s);

/* Device bytes a handle of this geometry will own (records, ancestry, state copies).
 * Host-only; validates like ola_create. */
ola_status ola_workspace_bytes(const ola_geometry* geom, uint64_t* out_bytes);

/* Create a decoder for one GDN layer of R requests.
 *   geom   : host pointer, copied.
 *   S_ctx  : device [R][H][d_v][d_k] fp32, the shared post-prefill state of each (request,
 *            head). Copied into the handle on `stream`; the caller may free it once the stream
 *            has reached this point.
 *   out    : host pointer that receives the handle (set to NULL on failure).
 * Allocates every buffer of ola_workspace_bytes on the current device. Step counter t = 0.
 * Errors: INVALID_ARG, UNSUPPORTED (geometry, or device is not sm_100), OOM, CUDA. */
ola_status ola_create(const ola_geometry* geom, const float* S_ctx, void* stream,
                      ola_handle* out);

/* One decode step (t := t + 1) for every request, beam and head.
 *   q, k       : device [R][B][H][d_k], in_dtype. q, k are used as given (no normalisation,
 *                no scaling).
 *   v          : device [R][B][H][d_v], in_dtype.
 *   g          : device [R][B][H] fp32, log decay (alpha = exp(g)).
 *   beta       : device [R][B][H] fp32, write strength.
 *   parent_idx : device [R][B] int32. Step 1: must be 0 (the shared state is the only
 *                parent). Later steps: index of the parent beam among the previous step's B
 *                beams, shared by all heads of the request. Out of range: clamped to 0 and
 *                OLA_ERR_BAD_PARENT is recorded (sticky).
 *   out_o      : device [R][B][H][d_v] fp32, o_t = S_t q_t (written, never read).
 * Errors: INVALID_ARG, CAPACITY (t == T_max; nothing launched), a sticky device error that
 * ola_get_error has returned (nothing launched), CUDA. */
ola_status ola_step(ola_handle h, const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const int32_t* parent_idx, float* out_o, void* stream);

/* ola_step with HOST buffers of the same layouts: copies the inputs into library-owned
 * device staging buffers (one cudaMemcpyAsync per tensor), runs the step, copies out_o
 * back, and returns after `stream` has finished (synchronous). Pinned host memory makes
 * the copies asynchronous DMA; pageable memory works but is slower. */
ola_status ola_step_host(ola_handle h, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const int32_t* parent_idx,
                         float* out_o, void* stream);

/* ola_step_host without waiting: pipelined decode from host buffers. The inputs are copied
 * in on a copy stream of the handle, the step runs on `stream` and out_o is copied back on a
 * second copy stream, so one call's copy-out overlaps the next call's copy-in (the host link
 * carries both directions at once). Two device staging sets are used in turn. Returns once the
 * work is queued. The host buffers of a call must stay valid, and out_o unread, until
 * ola_host_sync; they must be pinned for the copies to be asynchronous.
 * Errors: as ola_step; INVALID_ARG for NULL pointers; CUDA. */
ola_status ola_step_host_async(ola_handle h, const void* q, const void* k, const void* v,
                               const float* g, const float* beta, const int32_t* parent_idx,
                               float* out_o, void* stream);

/* Wait for every queued ola_step_host_async call (its copies and steps); then as
 * ola_get_error. */
ola_status ola_host_sync(ola_handle h);

/* Rewind to t = 0, keeping S_ctx, and clear the sticky device error. Stream-ordered on the
 * stream of the handle's last call (no host synchronisation): work queued before it still
 * runs, and the next ola_step must be queued on that stream or ordered after it. */
ola_status ola_reset(ola_handle h);

/* Current step t (0 .. T_max), or -1 for a NULL handle. Host-only. */
int32_t ola_current_step(ola_handle h);

/* Ancestry of the current beams: out[r][b][s] (device [R][B][t] int32) = the beam index of
 * the record that beam b's chain holds at step s+1 (out[r][b][t-1] == b). Stream-ordered.
 * Errors: INVALID_ARG (NULL, or t == 0), CUDA. */
ola_status ola_get_ancestry(ola_handle h, int32_t* out, void* stream);

/* Wait for the handle's queued work, then return its sticky device error (OLA_OK if none). */
ola_status ola_get_error(ola_handle h);

/* Record reclamation ("Scientific Impact Assessment: OneLA", §1: append-only transition
 * records over one shared post-prefill state, pruning through the parent-pointer ancestry
 * index). Finds the longest prefix of chain slots at which every live beam of every request
 * holds the same record (beam search that has converged), folds those records into S_ctx in
 * chain order (S <- alpha_j S + w_j k_j^T, the transition written with the record; fp32, and
 * the bf16 split of the tensor path is recomputed), moves the later records, chain rows and
 * ranks down by that many slots and decreases t by it. Later steps give the same outputs up to
 * rounding, and a decode can run past T_max while its beams keep converging. The current
 * step's own records are never folded (t stays >= 1). ola_get_ancestry afterwards returns the
 * chains without the folded slots, and ola_reset keeps the folded S_ctx. On the REPLAYSSM
 * path the folded records are raw tokens and are applied with the gated delta rule itself.
 *   out_folded : host int32, optional (NULL): number of folded steps (0 if none).
 * Synchronises `stream`, which must be the stream of the handle's previous calls (or ordered
 * after them). FullState handles keep every beam's state, so nothing is folded there: only the
 * ancestry rows of the shared slots are dropped and t lowered, which lets them decode past T_max
 * too (out_folded counts those slots).
 * Errors: INVALID_ARG (NULL handle), the sticky device error, CUDA. */
ola_status ola_compact(ola_handle h, int32_t* out_folded, void* stream);

/* Free every buffer of the handle (waits for its queued work first). NULL is a no-op.
 * The handle must not be used afterwards. */
ola_status ola_destroy(ola_handle h);

/* Shared post-prefill state from a prompt: for each (request, head), start from S = 0 and
 * apply the transition above to the prompt tokens p = 0..P-1 in order ("Scientific Impact
 * Assessment: OneLA", §1: one state derived from the shared prompt), in fp32.
 *   k    : device [R][P][H][d_k], in_dtype;   v : device [R][P][H][d_v], in_dtype
 *   g    : device [R][P][H] fp32 (log decay);  beta : device [R][P][H] fp32
 *   S_out: device [R][H][d_v][d_k] fp32 (written).
 * d_k, d_v in {16, 32, 64, 128, 256}; P >= 0 (P = 0 writes zeros).
 * d_k = d_v = 128 with a bf16 prompt (k, v 16-byte aligned) runs the chunked tensor-core form
 * (64 tokens per chunk, one CTA per (request, head)) and returns once it has finished, so that
 * a device-side wait that ran out is returned as OLA_ERR_TIMEOUT (such calls from several host
 * threads run one at a time: they share one device error word per device); every other shape
 * runs token by token on CUDA cores and returns after the launch (stream-ordered).
 * Errors: INVALID_ARG, UNSUPPORTED, OOM, TIMEOUT, CUDA. */
ola_status ola_prefill(int32_t R, int32_t H, int32_t d_k, int32_t d_v, int32_t P,
                       int32_t in_dtype, const void* k, const void* v, const float* g,
                       const float* beta, float* S_out, void* stream);

/* ------------------------------------------------------------------ allocation-free decode
 * Not from the pages: the paper has no counterpart of this entry point. It serves callers that
 * may not allocate device memory while they decode: servers whose device memory is reserved up
 * front by an arena or caching allocator (a cudaMalloc behind its back can fail once the arena
 * holds the device, or fragment it), plugins loaded into a host application that owns every
 * device allocation, and latency-critical loops that cannot afford the device-wide
 * synchronisation a cudaMalloc / cudaFree can imply.
 *
 * ola_decode_noalloc runs a whole T_max-step decode of one GDN layer on the fp32 CUDA-core
 * replay path (same results as ola_create + T_max x ola_step + ola_destroy with
 * path = REPLAY, math = FP32), without creating a handle and without allocating anything:
 *   geom        : host pointer; path must be OLA_PATH_REPLAY and math OLA_MATH_FP32; T_max is
 *                 the number of steps decoded; the geometry limits are those of ola_create.
 *   S_ctx       : device [R][H][d_v][d_k] fp32 shared state (read only), 16-byte aligned.
 *   q, k        : device [T_max][R][B][H][d_k] in_dtype;  v : device [T_max][R][B][H][d_v]
 *                 (16-byte aligned).
 *   g, beta     : device [T_max][R][B][H] fp32;  parent_idx : device [T_max][R][B] int32
 *                 (4-byte aligned); parents as for ola_step, step by step.
 *   out_o       : device [T_max][R][B][H][d_v] fp32 (written), 16-byte aligned.
 * The transient state (transition records, ancestry rows, error word) lives in one fixed
 * device array of OLA_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library, held by every GPU
 * that loads the library until the process exits. Problems needing more than that
 * (ola_noalloc_scratch_bytes) are rejected with OLA_ERR_SCRATCH_LIMIT, and bad geometry or
 * pointers with INVALID_ARG / UNSUPPORTED, before anything is queued. Every call shares the
 * array and leaves its contents behind (the call clears the error word itself); calls whose
 * work overlaps on the GPU (different streams, or several host threads) race on it and must be
 * serialised by the caller. The first call on each device resolves the array's device address
 * (a runtime query, no allocation); make that first call before any stream capture. The call
 * is synchronous: it waits for `stream` and returns the device error status (OLA_OK,
 * OLA_ERR_BAD_PARENT, ...) of this decode; on OLA_ERR_CUDA it has still waited for whatever
 * it had queued. */
#define OLA_NOALLOC_SCRATCH_BYTES (16u << 20)

uint64_t ola_noalloc_scratch_bytes(const ola_geometry* geom);

ola_status ola_decode_noalloc(const ola_geometry* geom, const float* S_ctx, const void* q,
                              const void* k, const void* v, const float* g, const float* beta,
                              const int32_t* parent_idx, float* out_o, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* OLA_H_ */
