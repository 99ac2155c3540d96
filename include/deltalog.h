/*
 * deltalog.h -- C ABI of libdeltalog, the DeltaLog decode step for
 * linear-attention recurrent state on NVIDIA B200 (sm_100a).
 *
 * What it computes.  Per (slot, head) the logical recurrent state
 * S_t in R^{d_k x d_v} of one of three operators (DeltaLog technical summary,
 * gist.science, section "Kernel implementation", operator list):
 *   GDN    S_t = a_t S_{t-1} + k_t b_t^T,  b_t = beta_t (v_t - a_t S_{t-1}^T k_t),
 *          o_t = S_t^T q_t                        (a_t scalar per head)
 *   KDA    S_t = diag(a_t) S_{t-1} + k_t b_t^T,
 *          b_t = beta_t (v_t - (diag(a_t) S_{t-1})^T k_t),  o_t = S_t^T q_t
 *   RWKV6  o_t = (S_{t-1} + diag(u) k_t v_t^T)^T r_t,
 *          S_t = diag(w_t) S_{t-1} + k_t v_t^T
 * is kept as a dense fp32 base Sbar plus a bounded log of compact factors
 * (a_i = k_i, b_i) with a log-decay snapshot Lam_i per entry (same summary,
 * section "Method -- core mechanism: base + log").  Steps 1..M-1 of each
 * cycle only append one entry; step M computes its output and writes the
 * full state back into Sbar, emptying the log ("append phase" / "merge
 * phase").  Every output equals the eager recurrence's up to rounding
 * (arXiv 2608.15533 abstract: the model sees the same dense state as eager
 * decoding).  dl_eager_step is the dense baseline that reads and writes the
 * whole state every token (summary, section "Problem: the state-update tax").
 *
 * Layouts (all C-contiguous, row-major, last index fastest):
 *   state      float  [B][H][d_k][d_v]     (d_v contiguous)
 *   q / r, k   in_dtype [B][H][d_k]
 *   v          in_dtype [B][H][d_v]
 *   o          in_dtype [B][H][d_v]
 *   log_decay  float  [B][H]       GDN: natural log of a_t (<= 0)
 *              float  [B][H][d_k]  KDA: log a_t per key; RWKV6: log w_t per key
 *   beta       float  [B][H]       GDN and KDA; must be NULL for RWKV6
 *   u          float  [H][d_k]     RWKV6 bonus (dl_set_bonus)
 * in_dtype is DL_F32 (float) or DL_BF16 (bfloat16, IEEE upper half).
 * Decays enter as natural logs: the library never divides by a cumulative
 * decay; every replay ratio is exp(Lam_t - Lam_i) <= 1.
 *
 * Ownership.  The caller owns every pointer it passes and the stream.  The
 * handle owns Sbar, the log, two small device staging sets for dl_step_host
 * and one copy stream, created by dl_create on the device current at that
 * time and released by dl_destroy.
 * Every call runs on that device (the caller's current device is restored).
 * All device-pointer calls are asynchronous on `stream` (a cudaStream_t, NULL
 * = legacy default stream): inputs must stay valid and outputs must not be
 * read until the stream reaches the call.  A handle must not be used from two
 * host threads at once, nor on two streams whose work overlaps.
 *
 * Errors.  Every int-returning call returns DL_OK (0) or a negative
 * dl_status; nothing aborts, throws or traps.  On an error the handle is
 * unchanged, except DL_ERR_CUDA after work was already queued.
 * dl_last_error() gives a message for the last failing call of this thread.
 */
#ifndef DELTALOG_H
#define DELTALOG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dl_handle* dl_t;

enum dl_op { DL_GDN = 0, DL_KDA = 1, DL_RWKV6 = 2 };
enum dl_dtype { DL_F32 = 0, DL_BF16 = 1 };

enum dl_status {
  DL_OK = 0,
  DL_ERR_ARG = -1,          /* null handle/pointer, bad size, misaligned pointer */
  DL_ERR_UNSUPPORTED = -2,  /* (op, d_k, d_v, dtype, M) not compiled in */
  DL_ERR_CUDA = -3,         /* a CUDA runtime call or kernel launch failed */
  DL_ERR_OOM = -4,          /* device or pinned allocation failed */
  DL_ERR_DEVICE = -5,       /* a kernel raised the handle's device error word */
  DL_ERR_STATE = -6         /* call not valid in the handle's current state */
};

/* Create a handle for B slots x H heads.  Supported: d_k, d_v in {64, 128},
 * 1 <= M <= DL_MAX_M, or M = DL_M_AUTO for dl_suggest_m's choice (read it
 * back with dl_merge_interval).  The base state starts at zero with an empty
 * log; the RWKV6 bonus starts at zero.  Pointers passed later must be aligned
 * to their element size (state pointers to 16 bytes).  M = 1 makes every step
 * a merge step (the deferred path then performs the eager schedule). */
#define DL_MAX_M 64
#define DL_M_AUTO 0
int dl_create(dl_t* out, int B, int H, int d_k, int d_v, int M, int op, int in_dtype);

/* Merge interval for an operator and head shape (no handle, no device).
 * The pages put the best M where the replay reads of a growing log balance
 * the saved dense writes (DeltaLog technical summary, gist.science, traffic
 * model).  Per (slot, head) and token, with S = 4 d_k d_v state bytes and e
 * log-entry bytes (a_i, b_i, Lam_i in their stored types), a cycle of M
 * tokens costs about
 *     f(M) = S/M + e (M-1)/M + rho (M-1)/2      (plus terms without M)
 * bytes: the merge write, the appended entries, and the replay of
 * 0 + 1 + ... + (M-1) entries at rho byte-equivalents each.  rho = e
 * c(op, d_k, d_v), where c is the replay cost per entry over its bytes as
 * measured on B200 for the square shapes (c = 1, pure traffic, for d_k !=
 * d_v).  Writes the M in [2, DL_MAX_M] that minimises f.  DL_ERR_ARG for an
 * unsupported op, shape or dtype, or a NULL M. */
int dl_suggest_m(int op, int d_k, int d_v, int in_dtype, int* M);

/* The handle's merge interval (the one chosen when created with DL_M_AUTO). */
int dl_merge_interval(dl_t h, int* M);

/* Free everything the handle owns.  Synchronises the handle's device first.
 * NULL is accepted and ignored. */
int dl_destroy(dl_t h);

/* Copy the dense state S [B][H][d_k][d_v] (device pointer) into Sbar and empty
 * the log: the next step starts a new merge cycle.  Sbar is the dense base
 * that holds the history up to the last merge point (DeltaLog technical
 * summary, gist.science, section "Method -- core mechanism: base + log",
 * item 1). */
int dl_load_state(dl_t h, const float* S, void* stream);

/* RWKV6 only: copy the bonus u [H][d_k] (device pointer). */
int dl_set_bonus(dl_t h, const float* u, void* stream);

/* One DeltaLog decode token for all B slots and H heads.  q is r for RWKV6.
 * With n entries in the log before the call (every slot holds n; see
 * dl_slot_load): if n + 1 < M the step appends (Sbar is read, never
 * written); if n + 1 == M it merges (Sbar <- S_t and the log empties).
 * These are the append and merge phases of the DeltaLog technical summary
 * (gist.science, section "Method -- core mechanism: base + log": for M-1
 * steps only compact factors and the current log-decay snapshot are
 * appended; every M steps base plus replayed log is written into the base
 * and the log reset).  Every step's output is computed from base + replayed
 * log, so it is the eager recurrence's (arXiv 2608.15533 abstract, fugumt.com:
 * the model observes the same dense state as in eager decoding).
 * Writes o [B][H][d_v].  All pointers are device pointers. */
int dl_step(dl_t h, const void* q, const void* k, const void* v,
            const float* log_decay, const float* beta, void* o, void* stream);

/* dl_step over a subset of the slots, in any order (a serving batch over a
 * state pool of B slots).  Batch row r (0 <= r < rows <= B) runs on slot
 * slot_idx[r]: q, k, v, o, log_decay and beta are [rows][H][...] in the
 * layouts above, slot_idx is a device int32 array [rows].  A negative index
 * marks a padding row: nothing is read or written for it, o included.  An
 * index >= B is skipped the same way and sets DL_DEVERR_SLOT_INDEX in the
 * device error word (dl_check_device).  Rows must name distinct slots
 * (undefined otherwise).  The step appends or merges every named slot
 * exactly like dl_step.
 * Held slots.  A live sequence that sits a token out (paused, waiting for a
 * tool call, preempted to let others run) is named as s | DL_SLOT_HOLD: its
 * row reads no input and writes no output, and its logical state stays
 * exactly as it was.  On an append the slot receives a null entry (a_n = 0,
 * b_n = 0 and Lam_n = Lam_{n-1}: nothing is added and its decay does not
 * advance) and its base is not touched; on a merge step its log is folded
 * into its base.  The serving integration the pages describe (DeltaLog
 * technical summary, gist.science, section "Main contributions", item 3: the
 * operators integrated into a vLLM-based serving stack) needs a sequence to
 * stay in the pool while it is absent from a batch.  A slot that a step names neither way receives no
 * log entry, so from then on its state is undefined until dl_slot_load: a
 * handle's live slots must each be in every step, active or held.
 * rows == 0 is a no-op.  A map has at most 65535 rows (DL_ERR_UNSUPPORTED
 * otherwise). */
#define DL_SLOT_HOLD 0x40000000
int dl_step_indexed(dl_t h, const int* slot_idx, int rows, const void* q, const void* k,
                    const void* v, const float* log_decay, const float* beta, void* o,
                    void* stream);

/* Prefill -> decode hand-off: run the operator's recurrence over a packed
 * batch of prompts and write each prompt's final state as its slot's base.
 * The pages' decode path starts from a dense base that holds the history up
 * to the last merge point (DeltaLog technical summary, gist.science,
 * "Method -- core mechanism: base + log"); the end of a prompt is such a
 * point.
 *   rows        prompts in the batch (0 <= rows <= B, at most 65535);
 *   slot_idx    device int32 [rows]: slot of row r (negative: skip the row),
 *               or NULL: row r runs on slot r; rows must name distinct slots;
 *   cu_seqlens  device int32 [rows + 1]: row r owns tokens
 *               [cu_seqlens[r], cu_seqlens[r + 1]) of the packed inputs
 *               (0 <= start <= end <= total, else the row is skipped and
 *               DL_DEVERR_SEQLEN is raised);
 *   total       tokens in the packed inputs;
 *   q, k, v, o  [total][H][d] in the input dtype, log_decay [total][H] (GDN)
 *               or [total][H][d_k], beta [total][H] (GDN/KDA, NULL for
 *               RWKV6): the layouts of dl_step with tokens in place of slots;
 *               o receives every token's output;
 *   flags       DL_PREFILL_ZERO_STATE: every row starts from S = 0 (a new
 *               sequence); 0: from the slot's current logical state (a
 *               continued or chunked prompt, or a state loaded from a cache).
 * Afterwards each named slot's base holds the state after its last token and
 * its log entries are cleared (dl_slot_load's convention), so dl_step
 * continues from it.  Other slots are untouched.  The outputs equal the
 * eager recurrence's token by token up to fp32 rounding with the recurrent
 * kernel, and up to the tf32 rounding of the products with the state with
 * the chunked ones (DL_OPT_PREFILL_KERNEL).  With total == 0 the input
 * pointers may be NULL. */
#define DL_PREFILL_ZERO_STATE 1
int dl_prefill(dl_t h, const int* slot_idx, int rows, const int* cu_seqlens, long long total, int flags,
               const void* q, const void* k, const void* v, const float* log_decay,
               const float* beta, void* o, void* stream);

/* Same as dl_step with HOST pointers (pinned or pageable): copies the inputs
 * into handle-owned device buffers, runs the step and copies o back.  Inputs
 * must stay valid, and o is valid, once `stream` has reached the call.  By
 * default every copy is ordered on `stream`.  With DL_OPT_HOST_PREFETCH set
 * the uploads run on the handle's own copy stream as soon as the call is made
 * (two staging sets alternate), overlapping the previous call's step and
 * download; the caller then promises that the host inputs are completely
 * written when it makes the call (not produced by work still queued on
 * `stream`).  When o is pinned host memory mapped into the device's address
 * space (cudaHostAlloc / cudaHostRegister with UVA), the step writes it
 * directly and no separate download is made. */
int dl_step_host(dl_t h, const void* q, const void* k, const void* v,
                 const float* log_decay, const float* beta, void* o, void* stream);

/* Eager dense baseline: read S_{t-1} from Sbar, write S_t back, every token:
 * the dense materialisation after every token that the DeltaLog technical
 * summary describes as the state-update tax (gist.science, section
 * "Problem: the state-update tax in linear-attention decoding").  Requires
 * every slot's log to be empty (DL_ERR_STATE otherwise; call dl_merge). */
int dl_eager_step(dl_t h, const void* q, const void* k, const void* v,
                  const float* log_decay, const float* beta, void* o, void* stream);

/* dl_eager_step over batch rows on the slots slot_idx[0..rows), with the
 * conventions of dl_step_indexed (padding rows, index errors, distinct
 * slots).  Slots not named, and held slots (DL_SLOT_HOLD), keep their
 * state. */
int dl_eager_step_indexed(dl_t h, const int* slot_idx, int rows, const void* q, const void* k,
                          const void* v, const float* log_decay, const float* beta, void* o,
                          void* stream);

/* Fold every slot's log into Sbar now (no output) and empty them; a no-op
 * when all logs are empty.  For an explicit flush or a checkpoint.  This is
 * the merge phase without a token (DeltaLog technical summary, gist.science,
 * section "Method -- core mechanism: base + log": the accumulated logical
 * state, base plus replayed log entries, written into the base). */
int dl_merge(dl_t h, void* stream);

/* Write the logical state (Sbar + replayed log) to S_out [B][H][d_k][d_v]
 * (device pointer) without changing the handle: the dense state the model
 * observes, equal to the eager decoder's (arXiv 2608.15533 abstract,
 * fugumt.com). */
int dl_read_state(dl_t h, float* S_out, void* stream);

/* Tuning options.  DL_OPT_STEP_KERNEL picks the kernel behind dl_step:
 *   DL_STEP_AUTO (default) and DL_STEP_REGISTER: the register-tile kernel
 *     (one CTA per slot-head and value tile), the only step kernel.
 * Returns DL_ERR_ARG for an unknown option or value. */
/* DL_OPT_HOST_PREFETCH (0 or 1, default 0): see dl_step_host.
 * DL_OPT_PDL (0 or 1, default 1): a register-tile step that follows an append
 * step of the same handle is launched as a programmatic dependent of the
 * previous kernel in the stream, so its blocks become resident while that
 * kernel drains.  Until that kernel has completed, the step reads nothing but
 * Sbar (written only by this handle's own launches, and never by an append):
 * its inputs, the slot map, the bonus and the log are read after it.  Kernels
 * of the caller between two dl_step calls (producing the next token's inputs,
 * say) are therefore safe with the option on.  Append steps allow their
 * successor to launch early; merge steps, dl_eager_step and dl_merge never
 * do. */
/* DL_OPT_VALUE_TILES (0 = automatic, 1, 2 or 4): value tiles per head of the
 * register-tile step kernel, i.e. how many CTAs split a head's d_v columns
 * (a split below 32 columns per tile falls back to fewer tiles; each tile
 * recomputes the head's key-side coefficients).  Automatic: 2 for d_v = 128
 * while the log holds fewer than 16 entries and the launch has at least two
 * (slot, head) units per SM, else 1. */
/* DL_OPT_LOG_B_BF16 (0 or 1, default 0): store the GDN/KDA value factors
 * b_i of the log in bf16 instead of fp32, 516 instead of 772 bytes per entry
 * for GDN d = 128 and 1024 instead of 1280 for KDA.  b_i is rounded to
 * nearest-even when appended; the current token's b_t enters its own output
 * and merge unrounded.  Every replayed or merged entry then carries a
 * relative error of at most 2^-9 in b_i, which feeds into later outputs and
 * into Sbar at each merge (outputs no longer equal the eager recurrence's up
 * to fp32 rounding only).  bf16-input handles only (DL_ERR_UNSUPPORTED
 * otherwise); a no-op for RWKV6, whose log already holds raw bf16 v_i.
 * Changeable only while the log is empty (DL_ERR_STATE otherwise). */
/* DL_OPT_LOG_LAM_F16 (0 or 1, default 0): store the per-key decay metadata of
 * KDA/RWKV6 log entries as each step's log-gates in fp16 instead of fp32
 * cumulative snapshots Lam_i: 1024 instead of 1280 bytes per entry for KDA
 * at d = 128 (768 with DL_OPT_LOG_B_BF16), 384 instead of 512 for RWKV6 at
 * d = 64.  The pages name the per-key metadata as the reason KDA and RWKV6
 * gain less than GDN (DeltaLog technical summary, gist.science, section
 * "Results").  Each kernel that reads a log rebuilds the fp32 snapshots
 * Lam_i = g_0 + ... + g_i in entry order from the staged gates; the current
 * token's own gate enters unrounded.  A rounded gate errs by at most 2^-11
 * of itself, so a snapshot errs by at most 2^-11 |Lam_i| and a decay factor
 * e^{Lam} by at most e^{Lam} |Lam| 2^-11 <= 2^-11/e of the state (outputs
 * then match the eager recurrence to a few 1e-4, not to fp32 rounding).
 * bf16-input handles only (DL_ERR_UNSUPPORTED otherwise); a no-op for GDN,
 * whose snapshot is one scalar per entry.  Changeable only while the log is
 * empty (DL_ERR_STATE otherwise). */
/* DL_OPT_PREFILL_KERNEL picks the kernel behind dl_prefill:
 *   DL_PREFILL_AUTO (default): the chunked kernel for bf16-input handles
 *     whose prompts average at least 16 tokens at d_k = d_v = 128 and 32
 *     at the other shapes;
 *     the recurrent kernel otherwise;
 *   DL_PREFILL_RECURRENT: the recurrence token by token, state in registers
 *     (every operator and dtype; outputs equal the eager recurrence's up to
 *     fp32 rounding);
 *   DL_PREFILL_CHUNKED: the chunk form on tensor cores (bf16-input handles
 *     only, DL_ERR_UNSUPPORTED otherwise): 32-token chunks, the WY form of
 *     the delta rule for GDN and KDA, per-key pair weights of KDA and RWKV6
 *     formed exactly on the SIMT lanes.  Each CTA keeps a whole head's state
 *     in tensor memory and runs the products with it as tcgen05 MMAs, for
 *     every head shape.  The products with the state are tf32, inside the
 *     bf16-input tolerance. */
enum dl_option {
  DL_OPT_STEP_KERNEL = 0,
  DL_OPT_HOST_PREFETCH = 1,
  DL_OPT_PDL = 2,
  DL_OPT_VALUE_TILES = 3,
  DL_OPT_LOG_B_BF16 = 4,
  DL_OPT_PREFILL_KERNEL = 5,
  DL_OPT_TEST_STALL_LOG = 6,
  DL_OPT_LOG_LAM_F16 = 7
};
enum dl_prefill_kernel { DL_PREFILL_AUTO = 0, DL_PREFILL_RECURRENT = 1, DL_PREFILL_CHUNKED = 2 };
enum dl_step_kernel { DL_STEP_AUTO = 0, DL_STEP_REGISTER = 1 };
int dl_set_option(dl_t h, int option, int value);

/* Which kernel the most recent dl_step / dl_step_host launched:
 * DL_STEP_REGISTER (DL_STEP_AUTO before the first step). */
int dl_last_step_kernel(dl_t h, int* kind);

/* Which kernel the most recent dl_prefill launched: DL_PREFILL_RECURRENT or
 * DL_PREFILL_CHUNKED (DL_PREFILL_AUTO before the first prefill). */
int dl_last_prefill_kernel(dl_t h, int* kind);

/* Number of entries currently in every slot's log (host-side counter, exact
 * in stream order). */
int dl_log_len(dl_t h, int* n);

/* Per-slot lifecycle for serving (admission, eviction, checkpoint of one
 * sequence while the other slots keep decoding).  Every slot keeps the
 * handle's log length n: instead of starting a cycle of its own, a slot that
 * is loaded or merged while n > 0 has its n log entries set to a_i = 0,
 * b_i = 0, Lam_i = 0.  Such entries add nothing to S_t, and Lam_i = 0 makes
 * the cumulative decay of the following entries and of the base start at
 * that point, so the slot's logical state is exactly the loaded (or merged)
 * one and every later dl_step stays one lockstep launch.  At the handle's
 * next merge step the slot merges with the rest, possibly after fewer than
 * M tokens of its own.
 *   dl_slot_load: set slot `slot`'s state to S [H][d_k][d_v] (device pointer;
 *     NULL = zeros, e.g. a fresh sequence) and clear its log entries.
 *   dl_slot_merge: fold slot `slot`'s log into its base now (no output) and
 *     clear its log entries; a no-op when n = 0.
 *   dl_slot_read: write slot `slot`'s logical state (base + replayed log) to
 *     S_out [H][d_k][d_v] (device pointer) without changing the handle.
 * All are asynchronous on `stream`; DL_ERR_ARG for a slot outside [0, B). */
int dl_slot_load(dl_t h, int slot, const float* S, void* stream);
int dl_slot_merge(dl_t h, int slot, void* stream);
int dl_slot_read(dl_t h, int slot, float* S_out, void* stream);

/* Allocation-free decode.  The pages have no counterpart to this call; it is
 * an interface for callers that cannot allocate device memory.  Some callers
 * cannot call cudaMalloc: a plugin inside an inference engine that hands out
 * every byte of device memory from its own pool, a process whose device
 * memory budget is fixed before it starts, or a latency-critical loop that
 * cannot take an allocation's implicit device synchronisation.  They cannot
 * create a handle, which allocates its base and log.  dl_decode_static runs T
 * DeltaLog decode tokens for all B slots and H heads on a dense state S that
 * the caller owns; the log lives in one fixed device array of
 * DL_STATIC_SCRATCH_BYTES (16 MiB), which every device that loads this
 * library holds until the process exits.  The call allocates nothing.
 *   op, B, H, d_k, d_v, in_dtype   as for dl_create; 1 <= M <= DL_MAX_M;
 *   S        device float [B][H][d_k][d_v], 16-byte aligned: the state before
 *            the first token on entry, after the last token on return;
 *   u        RWKV6 bonus [H][d_k] (device); ignored for GDN and KDA;
 *   T        tokens; 0 is a no-op;
 *   q (r for RWKV6), k, v, log_decay, beta, o   token-major: [T] followed
 *            by the dl_step layout of each (o receives every token's output);
 *   dev_err  NULL, or a device int (cleared by the caller) that the kernels
 *            OR their DL_DEVERR_* bits into; with NULL the bits go to a word
 *            inside the array, cleared at the start of each call and not
 *            reported.
 * Tokens 1..M-1 of every M-token cycle append to the log and token M merges
 * into S (dl_step's schedule, cycles counted from the call's first token); a
 * partial last cycle is folded into S at the end, so S is dense on return.
 * The outputs and S equal those of a handle loaded with S that runs the same
 * T dl_steps and then dl_merge.  The log of the B*H units must fit the
 * array: per unit m (d_k es + d_v eb) bytes of factors and Lam bytes of
 * snapshots, with m = max(M - 1, 1), es the input element size, eb = es for
 * RWKV6 and 4 otherwise, Lam = 4 round4(m) for GDN and 4 m d_k otherwise,
 * plus 256-byte alignment of each of the three regions and 256 bytes for the
 * error word.  (GDN at d = 128, bf16, M = 8 takes 5,408 bytes a unit: about
 * 3,100 units, e.g. B = 96 at H = 32.)  A larger request returns DL_ERR_ARG
 * and says how many bytes it needs.
 * The first call on a device looks the array's address up on that device
 * (and may load the library's device code there): make it before any stream
 * capture.  Every call uses the same array and finds the previous call's log
 * in it; nothing of it is read before this call writes it, except the error
 * word, which the call clears.  Calls whose work overlaps on the GPU (on
 * different streams, or from several host threads) race on the array: the
 * caller must order them.  Asynchronous on `stream`, on the current device. */
#define DL_STATIC_SCRATCH_BYTES (16u << 20)
int dl_decode_static(int op, int B, int H, int d_k, int d_v, int M, int in_dtype, float* S,
                     const float* u, int T, const void* q, const void* k, const void* v,
                     const float* log_decay, const float* beta, void* o, int* dev_err,
                     void* stream);

/* Bits of the device error word. */
enum dl_device_error {
  DL_DEVERR_WAIT_TIMEOUT = 1,  /* a bounded wait gave up (a log copy in a step: that unit wrote
                                  nothing; a tensor-core MMA in a chunked prefill: that row
                                  stopped and did not write its state).  A wait runs out only
                                  when the hardware did not finish work it was given within a
                                  second; treat the CUDA context as suspect afterwards */
  DL_DEVERR_SLOT_INDEX = 2,    /* a slot index >= B (indexed steps, dl_prefill) */
  DL_DEVERR_SEQLEN = 4         /* dl_prefill: a row's cu_seqlens range is invalid */
};

/* Read and clear the handle's device error word in one atomic step on
 * `stream`, then synchronise `stream`.  Returns DL_OK, or DL_ERR_DEVICE with
 * the word's bits in the message.  Bits raised later by work still running
 * on other streams stay in the word for the next call. */
int dl_check_device(dl_t h, void* stream);

/* Static text for a status code, and the last error message of this thread. */
const char* dl_strerror(int status);
const char* dl_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DELTALOG_H */
