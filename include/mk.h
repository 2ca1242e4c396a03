/*
 * mk.h -- C ABI of the persistent batch-1 decode megakernel for one B200 (sm_100a).
 *
 * What the library computes: one greedy decode step of a Llama-style decoder
 * (optionally with a top-k MoE FFN) for a single sequence, as ONE persistent
 * kernel with one block per SM whose blocks never exit mid-step and read, at
 * run time, a host-built instruction tensor that tells each block which
 * operation to run next.  The blocks synchronise among themselves on the
 * device instead of through kernel boundaries (Kittens VM summary page,
 * "Method"; Hyperkernel teardown, "What a megakernel buys").
 * Dependencies between instructions are global-memory counters.  Weight tiles
 * stream through a multi-stage shared-memory ring fed by TMA bulk copies, with
 * an L2 prefetch of the following weights (epic-kernel README, "Pipelining for
 * B200 bandwidth", "L2 prefetching overlapped with prior instructions").
 *
 * Conventions for every function:
 *  - Return value: MK_OK (0) or a negative MK_ERR_* code; nothing here calls
 *    exit() or abort().  mk_strerror() names a code.
 *  - Pointers documented as "device" are CUDA device addresses on the device
 *    that was current at mk_create(); "host" pointers are ordinary CPU memory.
 *  - A handle is not thread-safe: one call at a time per handle.
 *
 * Data layout (all row-major, the nn.Linear [out, in] convention):
 *   bf16 weights: embed/lm_head [vocab, hidden]; wq [n_q_heads*head_dim, hidden];
 *   wk, wv [n_kv_heads*head_dim, hidden]; wo [hidden, n_q_heads*head_dim];
 *   w_gate, w_up [ffn, hidden]; w_down [hidden, ffn]; router [n_experts, hidden];
 *   norm weights [hidden].
 *   KV cache (bf16, caller-owned): k_cache, v_cache [n_layers][n_kv_heads][max_seq][head_dim].
 *   Activations inside the library are fp32; logits are fp32 [vocab].
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ----------------------------------------------------------- */
#define MK_OK 0
#define MK_ERR_INVALID_ARG (-1)   /* bad config, null pointer, pos >= max_seq, token outside [0, vocab) */
#define MK_ERR_CUDA (-2)          /* a CUDA runtime call failed; mk_status.cuda_error holds the cudaError_t */
#define MK_ERR_NOT_RESIDENT (-3)  /* the one-block-per-SM cooperative grid cannot be co-resident */
#define MK_ERR_TIMEOUT (-4)       /* a bounded device wait ran out (dependency counter or smem ring) */
#define MK_ERR_BAD_INSTR (-5)     /* the device met an opcode or index outside the valid range */
#define MK_ERR_SCHEDULE (-6)      /* the host validator rejected the schedule */
#define MK_ERR_STOPPED (-7)       /* the stop word was set before or during the step */
#define MK_ERR_NO_SCHEDULE (-8)   /* mk_decode_step before mk_build_schedule */
#define MK_ERR_CAPACITY (-9)      /* a caller buffer is too small */
#define MK_ERR_UNSUPPORTED (-10)  /* shape outside what the kernels handle (see mk_create) */

/* ---- execution modes -------------------------------------------------------- */
#define MK_MODE_MEGAKERNEL 0        /* one persistent cooperative launch per step */
#define MK_MODE_MULTI_KERNEL 1      /* baseline: one plain launch per op and layer */
#define MK_MODE_MULTI_KERNEL_GRAPH 2/* baseline launches replayed from a CUDA graph */

/* ---- fault injection (host side; see mk_inject_fault) ------------------------ */
#define MK_FAULT_NONE 0
#define MK_FAULT_UNREACHABLE_WAIT 1 /* one instruction waits for a counter value no step reaches */
#define MK_FAULT_BAD_OPCODE 2       /* one instruction carries an opcode outside the table */
#define MK_FAULT_PRESET_STOP 3      /* the stop word is set before the launch */

/* Model shape.  n_experts = 0 selects the dense SiLU-gated FFN; otherwise each
 * layer's FFN is a top_k-of-n_experts MoE (top_k in {1, 2}, n_experts <= 64).
 * Supported (else MK_ERR_UNSUPPORTED): head_dim in {64, 128}; 1 to 4 query
 * heads per kv head; hidden <= 8192; hidden, ffn and n_q_heads*head_dim
 * multiples of 8 and at most 16384, and a width above 8192 must split into 2
 * equal parts of whole 8-element chunks.  tied_embeddings: lm_head may equal
 * embed (informational). */
typedef struct {
    int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    int n_experts, top_k;
    float rms_eps, rope_theta;
    int max_seq;
    int tied_embeddings;
} mk_config;

/* Device pointers to bf16 weights and the bf16 KV caches; all caller-owned and
 * kept alive for the handle's lifetime (the library reads them, and writes the
 * KV caches at the decoded position).  Per-layer arrays are HOST arrays of
 * n_layers device pointers; for MoE, w_gate/w_up/w_down have
 * n_layers * n_experts entries ([layer * n_experts + expert]) and router has
 * n_layers entries.  router may be NULL for dense models; the KV caches may
 * be NULL when n_layers == 0.  All device pointers must be 16-byte aligned.
 * With options.batch = B > 1 each cache holds B sequences' caches one after
 * the other ([B][n_layers][n_kv][max_seq][head_dim]). */
typedef struct {
    const void *embed, *lm_head, *final_norm;
    const void *const *attn_norm, *const *wq, *const *wk, *const *wv, *const *wo, *const *ffn_norm;
    const void *const *w_gate, *const *w_up, *const *w_down;
    const void *const *router;
    void *k_cache, *v_cache;
} mk_weights;

/* Schedule and kernel knobs.  Zero selects the default for every field except
 * l2_prefetch, prefetch_ahead and l2_head_start (-1 = default, 0 = off). */
typedef struct {
    int ring_stages;      /* shared-memory weight ring depth (default 3; 2 for dense head_dim-128 models
                             and for batch > 1) */
    int stage_bytes;      /* bytes per ring stage, multiple of 1024 (default 65536; 98304 for dense
                             head_dim-128 models and for batch > 1, when ring_stages is left at 0 too) */
    int rows_per_instr;   /* cap on GEMV rows per instruction (default and max 1024) */
    int kv_splits;        /* split-KV chunks per kv head (0 = default, at most SMs / n_kv_heads: at
                             head_dim 64 the count minimising a fitted model of attention plus merge
                             time at max_seq, 6 for 1152 positions; at head_dim 128 about one split
                             per 128 positions of max_seq; n_q_heads * kv_splits <= 2048) */
    int l2_prefetch;      /* bytes kept prefetched into L2 ahead of the TMA stream (-1 default) */
    int trace;            /* 1: record per-instruction globaltimer stamps (mk_get_trace) */
    int snapshots;        /* 1: record the residual stream after every layer (mk_get_hidden) */
    unsigned long long spin_limit_ns; /* bound on every device-side wait (default 2 s) */
    int mode;             /* MK_MODE_* */
    int n_sm;             /* blocks of the persistent grid (default: all SMs) */
    int prefetch_ahead;   /* consumers prefetch into L2 the weights of the instruction this many
                             places ahead in their queue (-1 default, 0 = off) */
    int prefetch_max_bytes; /* cap on the bytes prefetched per instruction (0 = default 1 MiB) */
    int attn_sm_ffn_permille; /* fused-FFN rows of a block that also runs an attention split of the
                             layer, per mille of an even share (0 = default 1000: even split; 950
                             measured slower on the Llama-1B shape) */
    unsigned long long serve_idle_ns; /* launch-once serving: the grid leaves after this long without a
                             request (default 60 s) */
    int general_kernel;   /* 1: always run the general kernel instantiation (ablations; default 0 picks the
                             specialised one when the schedule allows it) */
    int split_ffn;        /* 0 (default): each layer's FFN is one fused instruction per SM (up/gate rows,
                             then the matching columns of w_down, streamed from a transposed copy the
                             library keeps, added into the residual with atomics: fp32 summation order
                             varies between runs); 1: separate up/gate and down instructions, no copy,
                             bitwise reproducible.  The split form is also used whenever hidden > 8192
                             or 2 * hidden > stage_bytes */
    int l2_head_start;    /* when the loader issues the first stage of a dense fused-FFN or LM-head
                             instruction, it also prefetches into L2 this many ring stages of that
                             instruction's weights past the ring (0..64; -1 default, 0 = off), so the
                             stream is already moving when the instruction's dependency is met */
    const float *sm_speed; /* host array of n_sm_speed relative streaming speeds, one per block of the
                             grid (NULL = all equal).  The dense fused FFN's rows and the LM head's rows
                             are split in proportion, so blocks that stream slower on this GPU take fewer
                             rows.  Each speed must be finite and > 0, and n_sm_speed must equal the
                             grid's block count.  Read (copied) by mk_create and mk_plan; the caller may
                             free it afterwards */
    int n_sm_speed;
    int spec_experts;     /* MoE models with the fused FFN: 1 = speculative expert prediction.  After its
                             last QKV instruction of a layer each block applies the layer's router to the
                             attention input (the RMSNorm of the residual entering the layer, with the
                             attention norm weights, already in registers), and its loader streams the
                             first ring stages of its FFN slice of the predicted experts before the real
                             routing is known; on a miss those stages are dropped and the routed expert's
                             rows are streamed instead.  The result is the same either way.  2 = predict
                             the experts with the lowest scores instead (every prediction misses unless
                             all experts are selected; exercises the miss path).  0 (default) = off */
    int batch;            /* sequences decoded together per step (1..8; 0 = 1).  With batch B > 1 every
                             weight stage that reaches shared memory is applied to the B sequences' input
                             vectors before its slot is freed, so the weights cross HBM once per step for
                             all of them; attention, RoPE, the KV append and the argmax run per sequence.
                             Each sequence has its own KV cache (the caches are [B][n_layers][n_kv]
                             [max_seq][head_dim], sequence-major), token and position, stepped by
                             mk_decode_step_batch.  B > 1 needs a dense model with the fused FFN in
                             megakernel mode, hidden and n_q_heads*head_dim at most 2048 (B <= 8) or 4096
                             (B <= 4), and no serving or speculative prediction; otherwise
                             mk_create returns MK_ERR_UNSUPPORTED */
    int attn_merge;       /* where the kv splits of the split attention are merged (the combine step of
                             split-KV decoding: each split's partial output rescaled by its running max).
                             1 = every O-projection block merges all splits of every head while loading
                             its input, so the partials are read from L2 once per block; 2 = the last split
                             of each kv head to finish merges that head's splits once and writes the
                             attention output, which the O-projection blocks read as a plain vector (one
                             atomic arrival per split, one extra L2 round trip for the last one).  0
                             (default) = 2 when the partials that every block would read exceed 96 KB
                             (n_q_heads * kv_splits * head_dim * 4 bytes) and batch is 1, else 1.  2 with
                             batch > 1 returns MK_ERR_UNSUPPORTED */
    int ffn_early_stages; /* dense models with the fused FFN: the loader issues at most this many of a
                             block's FFN stages before the FFN's dependency is met (the rest wait for it),
                             so that the weight stream leaves HBM and L2 quiet while the small ops before
                             the FFN run their latency chain.  -1 = no limit; 0 (default) = 1 for hidden
                             <= 2048 at batch 1 or 2 when the block's FFN slice spans at least 4 ring
                             stages, else no limit; 1..64 = that many */
} mk_options;

/* Device status block, copied out by mk_get_status.  On a device-side error
 * the first failing wait records where it gave up. */
typedef struct {
    int code;             /* MK_OK or MK_ERR_TIMEOUT / MK_ERR_BAD_INSTR / MK_ERR_STOPPED / MK_ERR_CUDA */
    int sm;               /* block index that recorded the error */
    int instr;            /* index of the instruction in that block's queue */
    int opcode;
    int counter;          /* counter id waited on (-1: the shared-memory ring) */
    unsigned int observed, expected;
    int cuda_error;       /* cudaError_t for MK_ERR_CUDA */
} mk_status;

typedef struct mk_handle mk_handle;

/* Fill *out with the defaults described in mk_options. */
void mk_default_options(mk_options *out);

/* Create a handle: validates the config and pointers, allocates the library's
 * device buffers (instruction tensor, counters, fp32 activations, status) on
 * the current device and binds `cuda_stream` (a cudaStream_t, NULL = legacy
 * default stream).  Errors: MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED, MK_ERR_CUDA.
 * Source: the one-time host set-up before the persistent kernel's first launch
 * -- weights placed at the addresses the plan names, the kernel's buffers and
 * launch shape fixed (Hyperkernel teardown, "What is in the repository"); the
 * shapes it accepts are the Llama and Mixtral decoders of the epic-kernel
 * README ("3B model support", "Mixtral 8x7B MoE for batch-1 inference"). */
int mk_create(const mk_config *cfg, const mk_weights *w, const mk_options *opt, void *cuda_stream,
              mk_handle **out);

/* Build, validate and upload the instruction schedule (host work, done once).
 * Deterministic: the instruction words depend only on (config, options, SMs).
 * Errors: MK_ERR_SCHEDULE (validator), MK_ERR_CUDA.
 * Source: the instruction tensor each block reads at run time to learn which
 * op it runs next (Kittens VM summary page, "Method"); a schedule whose
 * grid-wide waits cannot deadlock and that keeps every SM busy across ops of
 * different shapes is one of the hard parts the Hyperkernel teardown names
 * ("What a megakernel buys"). */
int mk_build_schedule(mk_handle *h);

/* Copy the instruction tensor ([n_sm][max_instr][MK_INSTR_WORDS] int32, unused
 * slots zero) to host `buf` of `cap` words.  *n_words receives the size.
 * Errors: MK_ERR_NO_SCHEDULE, MK_ERR_CAPACITY (cap too small; *n_words is set).
 * Source: the same instruction tensor (Kittens VM summary page, "Method"),
 * exposed so that schedules can be checked on the host. */
#define MK_INSTR_WORDS 16
int mk_get_schedule(mk_handle *h, int32_t *buf, size_t cap, size_t *n_words, int *n_sm, int *max_instr);

/* One decode step: embeds `token` (or, if token < 0, the previous step's
 * on-device argmax), runs every layer at position `pos` (appending K/V at pos
 * and attending over 0..pos), writes fp32 logits to `logits_dev` (device,
 * [vocab], may be NULL) and, if `next_token_host` is not NULL, waits for the
 * step and stores the argmax there (lowest index on ties).  With
 * next_token_host == NULL the call only enqueues on the handle's stream, and
 * device-side errors surface at the next synchronous call or mk_get_status.
 * Positions must be stepped in order: pos reads cache entries 0..pos-1.
 * Errors: MK_ERR_INVALID_ARG, MK_ERR_NO_SCHEDULE, MK_ERR_TIMEOUT,
 * MK_ERR_BAD_INSTR, MK_ERR_STOPPED, MK_ERR_CUDA.
 * Source: one megakernel launch per call, the whole forward pass inside it
 * (Hyperkernel teardown, "A single kernel launch, read from the host": one
 * launch per call); the forward is the batch-1 decode step of the epic-kernel
 * README's models, the next-token choice the greedy argmax. */
int mk_decode_step(mk_handle *h, int32_t token, int32_t pos, float *logits_dev, int32_t *next_token_host);

/* One decode step of the options.batch sequences of the handle in one launch:
 * sequence b embeds tokens[b] (token < 0: its previous on-device argmax), runs
 * every layer at position pos[b] against its own KV cache (appending at pos[b],
 * attending over 0..pos[b]); positions may differ between sequences.  tokens
 * and pos are host arrays of batch entries (read before the call returns).
 * logits_dev: device [batch][vocab] fp32, may be NULL.  next_host: host array
 * of batch entries, or NULL to only enqueue (as mk_decode_step).  A batch-1
 * handle accepts this call too (the same step as mk_decode_step).
 * Errors: as mk_decode_step; MK_ERR_INVALID_ARG for a null array or a bad
 * token or position.
 * Source: a megakernel removes the launch gaps that dominate batch-1 decode,
 * while at larger batch the matrix products grow to hide them (Hyperkernel
 * teardown, "What a megakernel buys"); this is the small-batch variant of the
 * same step, each weight read from HBM once for every sequence of the batch. */
int mk_decode_step_batch(mk_handle *h, const int32_t *tokens, const int32_t *pos, float *logits_dev,
                         int32_t *next_host);

/* Residual stream after layer `layer` of the last step (0 = embedding,
 * n_layers = after the last layer) as fp32 [batch][hidden] into host
 * `out_host` (batch = options.batch, 1 by default).
 * Needs options.snapshots = 1.  Synchronises the stream.
 * Source: per-layer checks against a reference, the kind of correctness
 * evidence the Hyperkernel teardown asks a megakernel release to ship ("What a
 * megakernel buys": correctness checks good enough to trust the result). */
int mk_get_hidden(mk_handle *h, int layer, float *out_host);

/* MoE routing of `layer` in the last step: top_k expert ids and weights
 * (host arrays of top_k entries).  MK_ERR_INVALID_ARG for dense models.
 * Source: the router scoring and expert selection the epic-kernel README fuses
 * into its MoE instructions ("Mixtral 8x7B MoE for batch-1 inference"). */
int mk_get_router(mk_handle *h, int layer, int32_t *idx, float *w);

/* Speculative expert prediction (options.spec_experts > 0): the top_k experts
 * predicted for `layer` in the last step from the residual entering the layer
 * (host array of top_k entries, best first), to compare with mk_get_router.
 * Synchronises.  Entries are -1 for a layer that no block predicted (the
 * schedule gives the prediction to blocks that run a QKV instruction and an
 * FFN slice of the layer; with every block doing so, every layer is predicted).
 * MK_ERR_INVALID_ARG for dense models or with the option off.
 * Source: the instruction that predicts the top-2 experts from the
 * pre-attention residual while attention runs, so that the predicted experts'
 * weights are on their way before the router confirms them (epic-kernel README,
 * "Speculative expert prediction"). */
int mk_get_predicted_experts(mk_handle *h, int layer, int32_t *idx);

/* Dependency counters (uint32, monotone across steps) into host `out`.
 * Source: the blocks synchronise on the device instead of through kernel
 * boundaries (Hyperkernel teardown, "What a megakernel buys"); these are the
 * global-memory counters they synchronise on. */
int mk_get_counters(mk_handle *h, uint32_t *out, size_t cap, size_t *n);

/* Per-counter increment per step, as planned by the scheduler (host `out`). */
int mk_get_counter_increments(mk_handle *h, uint32_t *out, size_t cap, size_t *n);

/* Copy the device status block (synchronises the stream).
 * Source: the control block with a watchdog word, a stop word and bounds
 * flags, and a host that reports a failed step instead of a number
 * (Hyperkernel teardown, "Hardware fault detection and replanning"). */
int mk_get_status(mk_handle *h, mk_status *out);

/* Trace stamps of the last step: [n_sm][max_instr][32] uint64 globaltimer ns,
 * zero where not reached.  Consumer warps: 0 instruction reached, 1 dependency
 * satisfied, 2 input vector ready, 3 first stage full, 4 main stages consumed
 * (the fused FFN's up/gate rows), 5 done and signalled.  Loader warp: 6 first
 * stage issued, 7 last stage issued.  Then for the instruction's first 8 ring
 * stages s: 8 + s consumer thread 0's wait for the stage returned, 16 + s its
 * share of the stage consumed, 24 + s the loader issued the stage.  Needs
 * options.trace = 1.
 * Source: the per-instruction timing trace the epic-kernel README records for
 * its SM-occupancy and HBM-utilisation plots (its profiling instructions). */
int mk_get_trace(mk_handle *h, uint64_t *out, size_t cap, size_t *n);

/* Clear counters, epoch, status and stop word and re-upload the schedule
 * (undoes mk_inject_fault).  Use after any failed step. */
int mk_reset(mk_handle *h);

/* ---- launch-once serving ---------------------------------------------------
 * The persistent grid stays resident across decode steps: no launch per step.
 * mk_serve_start launches it on the handle's stream (megakernel mode, schedule
 * built).  Each mk_serve_step writes (token, pos) to a mailbox in pinned host
 * memory and waits, bounded like mk_decode_step, until the grid has run that
 * step and posted its next token (token < 0: the previous step's argmax).
 * Logits go to the device buffer given at start (or the internal one); read
 * them from another stream after mk_serve_step returns.  mk_serve_stop asks the
 * grid to leave and waits for it.  The grid also leaves by itself after
 * serve_idle_ns without a request; the next mk_serve_step then returns
 * MK_ERR_STOPPED and mk_serve_start may be called again.  While serving, the
 * calls that touch the device (step, reset, getters, fault injection, schedule
 * rebuild) return MK_ERR_INVALID_ARG; mk_destroy stops the grid first.
 * Counters and KV positions continue across the serving and per-launch paths
 * (same epoch rule).  This is the launch-once, ring-fed server loop of the
 * Hyperkernel teardown ("A single kernel launch, read from the host").
 * Errors: MK_ERR_INVALID_ARG, MK_ERR_STOPPED, MK_ERR_TIMEOUT, MK_ERR_BAD_INSTR,
 * MK_ERR_CUDA. */
int mk_serve_start(mk_handle *h, float *logits_dev);
int mk_serve_step(mk_handle *h, int32_t token, int32_t pos, int32_t *next_token_host);
int mk_serve_stop(mk_handle *h);

/* Host-side fault injection for tests: MK_FAULT_* (see above).  The fault
 * applies from the next step until mk_reset.  `arg` selects the block for
 * instruction faults. */
int mk_inject_fault(mk_handle *h, int kind, int arg);

/* Device-side step time of the last megakernel launch in ns (CUDA events on
 * the handle's stream); synchronises. */
int mk_last_step_ns(mk_handle *h, double *ns);

const char *mk_strerror(int code);
void mk_destroy(mk_handle *h);

/* ---- standalone ops ------------------------------------------------------------------- */

/* Bytes of workspace mk_attention_decode needs: n_q_heads * splits * (head_dim + 2) floats. */
size_t mk_attention_workspace_bytes(int n_q_heads, int head_dim, int splits);

/* GQA decode attention of one layer, as one op (two plain launches on
 * `stream`, a cudaStream_t or NULL): for query head h and its kv head
 * g = floor(h / (n_q_heads / n_kv_heads)),
 *   out[h] = softmax_j(q[h] . K[g][j] / sqrt(head_dim)) V[g][j],  j in [0, n_pos)
 * (the decode attention step of the Llama decoder the megakernel pages target;
 * the sequence is split into `splits` chunks whose partial softmax states are
 * merged by the log-sum-exp rule, "split-KV").
 * q: device fp32 [n_q_heads][head_dim], already rotated.  k_cache, v_cache:
 * device bf16 [n_kv_heads][max_seq][head_dim], 16-byte aligned.  out: device
 * fp32 [n_q_heads][head_dim].  workspace: device, at least
 * mk_attention_workspace_bytes(...) bytes, caller-owned, overwritten.
 * head_dim in {64, 128}; 1..4 query heads per kv head; 1 <= n_pos <= max_seq;
 * splits >= 1 (splits beyond n_pos leave empty chunks, which merge to
 * nothing).  Enqueues only.  Errors: MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED,
 * MK_ERR_CAPACITY (workspace too small), MK_ERR_CUDA. */
int mk_attention_decode(const float *q, const void *k_cache, const void *v_cache, int n_q_heads, int n_kv_heads,
                        int head_dim, int n_pos, int max_seq, int splits, float *out, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Size of the device-resident scratch of mk_attention_decode_noalloc: 1 MiB,
 * i.e. n_q_heads * splits * (head_dim + 2) <= 262144 floats. */
#define MK_ATTENTION_NOALLOC_SCRATCH_BYTES ((size_t)1 << 20)

/* mk_attention_decode for callers that cannot allocate device memory: the
 * same computation, arguments and errors, but no workspace argument.  It is
 * for code that must not call cudaMalloc, for example a host whose device
 * memory is owned by another allocator or pool, or a latency-critical decode
 * loop where an allocation (and the device synchronisation it can imply) is
 * not allowed.  This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine.  The pages describe no counterpart for it.
 *  - Its split partials live in one fixed device array of
 *    MK_ATTENTION_NOALLOC_SCRATCH_BYTES inside the library, present on every
 *    GPU that loads the library until the process exits; a call whose
 *    n_q_heads * splits * (head_dim + 2) floats exceed it returns
 *    MK_ERR_CAPACITY.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current, and again after the device's
 *    context has changed, e.g. after cudaDeviceReset); make that first call
 *    before any stream capture.
 *  - All calls share the array: calls that overlap on the GPU (for example on
 *    two streams at once) race and give wrong results; serialise them.  Each
 *    call writes every slot it reads, so no clearing is needed between calls. */
int mk_attention_decode_noalloc(const float *q, const void *k_cache, const void *v_cache, int n_q_heads,
                                int n_kv_heads, int head_dim, int n_pos, int max_seq, int splits, float *out,
                                void *stream);

/* ---- host-only planning (no GPU needed) ---------------------------------------- */

/* Plan the schedule for `n_sm` blocks without a device: writes the instruction
 * tensor ([n_sm][max_instr][MK_INSTR_WORDS]) to `buf` (cap words), the
 * per-SM instruction counts to `n_instr` (n_sm entries) and the per-step
 * increment of every counter to `ctr_inc` (ctr_cap entries).  Runs the
 * validator.  Errors: MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED, MK_ERR_CAPACITY,
 * MK_ERR_SCHEDULE. */
int mk_plan(const mk_config *cfg, const mk_options *opt, int n_sm, int32_t *buf, size_t cap, int *max_instr,
            int32_t *n_instr, uint32_t *ctr_inc, size_t ctr_cap, int *n_counters);

/* Execute a planned schedule on the host under a seeded random interleaving of
 * the blocks (an instruction may run once its counter has reached its target)
 * for `steps` steps.  Returns MK_OK when every instruction ran and every
 * counter ends at steps * its increment, MK_ERR_SCHEDULE on a deadlock or a
 * count mismatch.  *executed receives the number of instructions run. */
int mk_simulate(const int32_t *buf, int n_sm, int max_instr, const int32_t *n_instr, const uint32_t *ctr_inc,
                int n_counters, int steps, uint64_t seed, long long *executed);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
