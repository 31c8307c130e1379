/*
 * gdr.h -- C ABI of libgdr, the B200 (sm_100a) gated delta-rule library.
 *
 * The operation.  Per (batch, head) the library carries a state
 * S in R^{dk x dv} (fp32) through the tokens t = 0 .. T-1:
 *
 *     S~_t = Diag(g_t) S_{t-1}                      (decay of the old state)
 *     x_t  = S~_t^T k_t                             (readout at the key)
 *     S_t  = S~_t - a_t x_t^T + c_t v_t^T           (erase, then write)
 *     o_t  = S_t^T (scale * q_t)                    (readout after the update)
 *
 * and the five variants choose g, a and c:
 *
 *   GDR_DELTANET        g = 1                 a = c = beta_t k_t
 *   GDR_GATED_DELTANET  g = alpha_t (scalar)  a = c = beta_t k_t
 *   GDR_KDA             g in R^{dk}           a = c = beta_t k_t
 *   GDR_GDN2            g in R^{dk}           a = b_t (.) k_t,  c = w_t (.) k_t
 *   GDR_KLA             g = alpha_t (scalar)  a = c = beta_t k_t with
 *                                             beta_t = eta_t / (||k_t||^2 + eps)
 *
 * Sources: "Kaczmarz Linear Attention" (gist.science/ja/paper/2605.08587),
 * sections "problem definition" and "KLA update rule" (decayed state, residual
 * e_t = v_t - S~^T k_t, update S_t = S~ + beta_t k_t e_t^T, Kaczmarz step) and
 * section "implementation" (KLA keeps the state shape and the chunkwise solver
 * of Gated DeltaNet and only changes the diagonal coefficient matrix);
 * "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 * (ai-auto-bdv.pages.dev/blog/arxiv-260522791/), sections "what is new" and
 * "technical core" (channel-wise decay of KDA; separate channel-wise erase
 * gate b_t and write gate w_t; the chunkwise WY algorithm with the decay
 * absorbed into asymmetric erase factors).  The GDN-2 form above is the
 * reading of that page's garbled formula that reduces to KDA when
 * b_t = w_t = beta_t, as the page states it must.
 *
 * Conventions for every entry point:
 *  - `variant`, `dtype` and the returned status are plain ints carrying the
 *    values of gdr_variant_t, gdr_dtype_t and gdr_status_t below, so that the
 *    ABI is the same for C callers and for foreign-function bindings; `variant`
 *    may carry the GDR_RAW_INPUTS flag.  `stream` is a cudaStream_t.
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no device memory, keeps no pointer after the call returns and
 *    never synchronises: work is enqueued on `stream` (a cudaStream_t passed as
 *    void*; NULL means the legacy default stream) and the call returns.
 *  - Layouts are dense and row-major: q, k [B,T,H,dk]; v, o [B,T,H,dv];
 *    per-token scalars [B,T,H]; per-token channel vectors [B,T,H,dk];
 *    states [B,H,dk,dv].  q, k, v, o use the I/O dtype; all gates and the
 *    states are fp32.
 *  - Every tensor pointer must be 16-byte aligned.
 *  - Decay is passed in log space: log_g = log(g) <= 0 (the chunked kernels
 *    need cumulative log-decay).
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call launches nothing and returns a status other than GDR_OK.
 *    gdr_last_error() then gives a one-line reason (thread-local).
 *  - A launch failure is reported as GDR_ERR_CUDA.  Faults inside a kernel
 *    surface, as usual in CUDA, at the caller's next synchronisation.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_DELTANET = 0,
    GDR_GATED_DELTANET = 1,
    GDR_KDA = 2,
    GDR_GDN2 = 3,
    GDR_KLA = 4
} gdr_variant_t;

/*
 * Raw-input mode: OR this flag into `variant` (of any entry point) to pass q,
 * k, beta and the gates as raw projections and logits; the kernels then apply
 * the input transforms on their load paths instead of the caller doing a
 * separate elementwise pass:
 *   q <- q / max(||q||, 1e-6) and k <- k / max(||k||, 1e-6) per (token, head)
 *        (KLA's keys are left as they are: its Kaczmarz step
 *        eta / (||k||^2 + eps) already carries their norm);
 *   beta (eta for KLA), erase_b, write_w <- sigmoid of the value passed;
 *   log_g <- -softplus of the value passed, so that g = sigmoid(-x) in (0, 1).
 * These are the key normalisation and gate activations of the pages' layers
 * ("Kaczmarz Linear Attention", KLA update rule: beta_t = eta_t/(||k_t||^2 +
 * eps) with eta a gate; ablations: keys normalised), applied to the raw
 * activations.  Shapes, dtypes and layouts are unchanged.
 */
#define GDR_RAW_INPUTS 0x100

typedef enum {
    GDR_F32 = 0,   /* q, k, v, o in fp32 */
    GDR_BF16 = 1   /* q, k, v, o in bf16 */
} gdr_dtype_t;

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,   /* NULL where required, non-positive size, bad enum */
    GDR_ERR_UNSUPPORTED = 2,   /* valid request this build has no kernel for */
    GDR_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    GDR_ERR_CUDA = 4,          /* a CUDA launch or driver call failed */
    GDR_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (see gdr_device_status) */
    GDR_ERR_RANGE = 6          /* a chunked-kernel operand left its representable range */
} gdr_status_t;

/* Forward-call tensors.  Unused entries are NULL. */
typedef struct {
    const void *q;               /* [B,T,H,dk] I/O dtype */
    const void *k;               /* [B,T,H,dk] I/O dtype */
    const void *v;               /* [B,T,H,dv] I/O dtype */
    const float *beta;           /* [B,T,H]: beta_t (DeltaNet, GDN, KDA) or eta_t (KLA); GDN-2: unused */
    const float *log_g;          /* [B,T,H] (GDN, KLA) or [B,T,H,dk] (KDA, GDN-2); DeltaNet: unused */
    const float *erase_b;        /* [B,T,H,dk] GDN-2 only */
    const float *write_w;        /* [B,T,H,dk] GDN-2 only */
    const float *initial_state;  /* [B,H,dk,dv] or NULL for zeros */
    float *final_state;          /* [B,H,dk,dv] or NULL; may be the same buffer as initial_state */
    void *o;                     /* [B,T,H,dv] I/O dtype, written for every token */
} gdr_fwd_args_t;

/*
 * Bytes of device workspace gdr_forward_chunked uses for this problem and
 * `chunk` choice: for the chunked path (chunk 0 or 65 with bf16
 * I/O and dk = 128) B * H * ceil(T/64) records of 56 KB + 8 KB per 64 value
 * columns, plus 16 bytes (scalar decay: DeltaNet, Gated DeltaNet, KLA) or
 * 512 bytes (channel decay: KDA), plus 24 KB per 64 value columns for GDN-2;
 * 0 for every other path.  When few sequences of many chunks would leave
 * most of the device idle (B * H small, dv = 128, T >= 4033), the carry runs
 * in segments and the size adds their transition maps and start states
 * and, where the carry with outputs is cut finer than the maps, the maps'
 * snapshots at the part starts (fp32, a few to a few tens of MB).  The workspace is caller-owned scratch, overwritten by
 * every call; its contents are not needed after the call completes on the
 * stream.
 */
size_t gdr_forward_workspace_size(int variant, int dtype, int B, int T, int H,
                                  int dk, int dv, int chunk);

/*
 * Whole-sequence forward of B sequences of T tokens and H heads.
 *
 * chunk selects the algorithm:
 *   0  automatic: the chunked path when it covers the case and the workspace
 *      is at least gdr_forward_workspace_size() bytes, else the per-token
 *      kernel;
 *   1  the per-token kernel (fp32 state in registers, exact fp32 arithmetic,
 *      any supported shape; the path used for fp32 I/O);
 *   65 the chunked path (C = 64 tokens per chunk, tcgen05 tensor cores with
 *      TMEM accumulators fed by TMA): a chunk-parallel preparation kernel (the
 *      S-independent products of every chunk, into the workspace) then the
 *      sequential carry kernel: all five variants with bf16 I/O and dk = 128;
 *      needs the workspace.  Where the carry's B * H CTAs leave SMs idle it
 *      reschedules: for few long sequences, segment maps, a chain of segment
 *      start states, then the segments (or finer parts, see
 *      gdr_forward_segment_parts) in parallel; for a mid-size B * H,
 *      the sweep cut in two, with the second part's preparation beside the
 *      first part's carry.  Its kernels are chained on `stream` by
 *      programmatic dependent launch; the call returns after enqueueing them,
 *      like every other path.
 *   64 is reserved (a one-kernel chunked path without workspace, not built:
 *      GDR_ERR_UNSUPPORTED).
 * A chunk value whose path does not cover the case returns GDR_ERR_UNSUPPORTED.
 * Shapes: B, T, H >= 0; dk in {64, 128}; dv in {64, 128}.  T = 0 copies
 * initial_state to final_state (or clears it); B * H = 0 does nothing.
 * eps is used by KLA only; scale multiplies q.  workspace must be 16-byte
 * aligned; it may be NULL (with workspace_bytes ignored) for paths that use none.
 */
gdr_status_t gdr_forward_chunked(int variant, int dtype, int B, int T, int H, int dk, int dv,
                                 const gdr_fwd_args_t *args, float eps, float scale, int chunk,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward for callers that cannot allocate device memory at call time: a
 * serving runtime whose device memory is planned up front and that forbids
 * allocation on its request path, or a host program that drives this
 * library without a device allocator of its own.  It runs the
 * chunked path (chunk = 65 of gdr_forward_chunked) with the library's own
 * fixed scratch instead of a caller workspace, and allocates nothing.  The
 * pages have no counterpart to this entry point; it is a deployment
 * convenience.
 *
 * Arguments, layouts and results are those of gdr_forward_chunked.  It covers
 * the five variants with bf16 I/O, dk = 128, dv in {64, 128}; anything else
 * returns GDR_ERR_UNSUPPORTED.
 *
 * The fixed scratch is a 32 MiB device array in the library's device image:
 * every GPU that loads the library holds it until the process exits.  A call
 * needs B * H * ceil(T / 64) records (one per sequence, head and 64-token
 * chunk), and they must fit in the array: at most 32 MiB / record bytes,
 * i.e. 455 records at dv = 128 (511 at dv = 64) for DeltaNet, Gated DeltaNet
 * and KLA, 451 (508) for KDA, 271 (370) for GDN-2.  Larger problems return
 * GDR_ERR_UNSUPPORTED with the needed and available bytes and that limit in
 * gdr_last_error().  For few long sequences gdr_forward_chunked runs the
 * carry in segments, whose maps need room beside the records; where that room
 * is not left in the array, this call runs the unsegmented sweep instead (the
 * same results, a longer sequential carry).
 * The array's device address is looked up for the CURRENT device, so the
 * current device must be the device that owns `stream`.  The first call on
 * each device does that lookup (and may load the library's device code);
 * make that first call before any stream capture.  All calls share the array
 * and each call rewrites what it uses before reading it, so nothing needs
 * clearing; calls whose execution overlaps on the GPU (different streams, or
 * different host threads) race on the array and must be serialised by the
 * caller.
 */
gdr_status_t gdr_forward_chunked_noalloc(int variant, int dtype, int B, int T, int H, int dk, int dv,
                                         const gdr_fwd_args_t *args, float eps, float scale, void *stream);

/*
 * One recurrent decode token for N independent sequences and H heads: the
 * same per-token update as the forward ("Kaczmarz Linear Attention", KLA
 * update rule: decay, residual at the key, erase and write; the GDN-2 form
 * read as in the top comment), applied once to a state kept in device memory.
 * q, k [N,H,dk]; v, o [N,H,dv] (I/O dtype); beta [N,H]; log_g [N,H] or
 * [N,H,dk]; erase_b, write_w [N,H,dk]; state [N,H,dk,dv] fp32, read and
 * updated in place.  Gate roles as in gdr_fwd_args_t.  One kernel launch;
 * no workspace; validation and errors as for the forward.
 */
gdr_status_t gdr_decode_step(int variant, int dtype, int N, int H, int dk, int dv,
                             const void *q, const void *k, const void *v,
                             const float *beta, const float *log_g,
                             const float *erase_b, const float *write_w,
                             float *state, void *o, float eps, float scale, void *stream);

/* Backward-call gradients (outputs, caller-owned device memory).  Unused entries are NULL. */
typedef struct {
    void *dq;                 /* [B,T,H,dk] I/O dtype */
    void *dk;                 /* [B,T,H,dk] I/O dtype */
    void *dv;                 /* [B,T,H,dv] I/O dtype */
    float *dbeta;             /* [B,T,H]: d beta, or d eta for KLA; GDN-2: unused */
    float *dlog_g;            /* [B,T,H] (GDN, KLA) or [B,T,H,dk] (KDA, GDN-2); DeltaNet: unused */
    float *d_initial_state;   /* [B,H,dk,dv], or NULL when not wanted */
    float *d_erase_b;         /* [B,T,H,dk], GDN-2 only */
    float *d_write_w;         /* [B,T,H,dk], GDN-2 only */
} gdr_bwd_grads_t;

/*
 * Bytes of device workspace gdr_backward needs (0 for a case it does not
 * cover): the forward's records, the reverse carry's records (B * H *
 * ceil(T/64) of each), every chunk's start state (dk * dv, fp16; fp32 for
 * KDA) and end-state gradient (dk * dv, fp32), plus two states; for few long sequences (where the
 * forward's carry runs in segments) also the segment maps and start states
 * its two carries share.  The segmenting reads the current device's SM
 * count, so query the size on the device that runs the call.
 */
size_t gdr_backward_workspace_size(int variant, int dtype, int B, int T, int H, int dk, int dv);

/*
 * Gradients of  <d_o, o> + <d_final_state, S_T>  with respect to the
 * forward's inputs, for the forward that `args` describes (its o and
 * final_state are not used): the gate-aware backward that keeps the
 * chunkwise structure ("Gated DeltaNet-2: Decoupling Erase and Write in
 * Linear Attention", technical core), for all five variants with bf16 I/O,
 * dk = 128 and dv in {64, 128}.  With S
 * the state and dS its gradient, per 64-token chunk:
 *     forward   E = U' - W S0,  O = Qg S0 + P E,  S_C = Gamma_C S0 + Kt^T E
 *     backward  dE = Kt dS + P^T dO,  dS0 = Gamma_C dS + Qg^T dO - W^T dE
 * ("Kaczmarz Linear Attention", KLA update rule and implementation: the
 * chunkwise solver of Gated DeltaNet with KLA's diagonal step).  It re-runs
 * the forward's chunk products and carry (keeping every chunk's start state),
 * runs the dS recurrence through the same carry kernel over the chunks in
 * reverse (both carries in segments for few long sequences, as the
 * forward's), then computes every chunk's q, k, v and gate gradients in
 * parallel; for KDA the chunk products take the channel decay element by
 * element, factored around the chunk's middle token as the forward's are
 * (so the forward's GDR_ERR_RANGE check covers them too), and dlog_g is per
 * channel.  KLA's d eta includes the path through its Kaczmarz step
 * eta / (||k||^2 + eps).  d_o [B,T,H,dv] in the I/O dtype (required);
 * d_final_state [B,H,dk,dv] fp32 or NULL (zero).  The tensor-core carries use
 * fp16 operands with fp32 accumulation, like the forward's chunked path: the
 * gradients match an exact backward to a few 1e-3 of their RMS (measured
 * worst cases: d log g up to 1.7e-2 on long channel-decay sequences; GDN-2's gate
 * gradients, which the carries' fp16 rounding reaches in proportion to the
 * terms they are built from, ~5e-4 of the largest gradient of a chunk); the
 * gradients are rescaled internally by a power of two so that d_o's range
 * does not matter.  workspace: at least gdr_backward_workspace_size() bytes,
 * 16-byte aligned, overwritten.  For GDN-2 the records' state-free terms
 * (P^d V, D~^T V) do not enter the dS recurrence, and the chunk-local kernel
 * also returns d erase_b and d write_w.  The raw-input mode (GDR_RAW_INPUTS),
 * fp32 I/O and dk = 64 return GDR_ERR_UNSUPPORTED.  T = 0 gives
 * d_initial_state = d_final_state.  Validation and errors as for the
 * forward; a reverse-record operand beyond the fp16 range is reported as
 * GDR_ERR_RANGE by gdr_device_status().
 */
gdr_status_t gdr_backward(int variant, int dtype, int B, int T, int H, int dk, int dv,
                          const gdr_fwd_args_t *args, const void *d_o, const float *d_final_state,
                          const gdr_bwd_grads_t *grads, float eps, float scale,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * Kernel launches one gdr_forward_chunked call with these arguments makes
 * (0 if the call would be rejected), and a short name of the kernel that runs
 * ("chunk64_split", "token_f32io", "token_bf16io", or "none").
 * Host-only, no GPU work.  The chunked path makes 2 launches, or 4 when
 * it reschedules (segmented or pipelined sweep); that choice reads the
 * current device's SM count, and with no device present it is always 2.
 */
int gdr_forward_launches(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk);
const char *gdr_forward_kernel_name(int variant, int dtype, int B, int T, int H, int dk, int dv,
                                    int chunk);

/*
 * How the chunked path schedules B sequences of T tokens and H
 * heads on a device with `sms` SMs (host-only; no device is queried, so it
 * serves to inspect a plan for any device).  Writes
 *   *segments        the carry's segments per sequence (1: not segmented),
 *   *segment_chunks  64-token chunks per segment,
 *   *split_chunk     the chunk where the pipelined sweep cuts each sequence
 *                    (0: serial sweep; only when not segmented).
 * Segmenting needs dv = 128, at least 64 chunks and floor(sms / (B * H))
 * large enough for three segments; the pipelined sweep needs at least 16
 * SMs beside the carry's B * H and is taken where its cost model expects a
 * gain.  B * H = 0 plans one segment and no cut.  Returns
 * GDR_ERR_INVALID_ARG for an unknown variant, dv not in {64, 128}, a
 * negative size or a NULL output.
 */
gdr_status_t gdr_forward_plan(int variant, int B, int T, int H, int dv, int sms, int *segments,
                              int *segment_chunks, int *split_chunk);

/*
 * The second phase of a segmented plan (same arguments and errors as
 * gdr_forward_plan).  The segment maps come from a first phase of about two
 * CTAs per segment; the carry with outputs needs one CTA per part, so it may
 * cut each sequence finer, into *parts parts of *part_chunks chunks (the last
 * one ragged), each starting from the map and offset of its segment after the
 * chunks before it.  Without segmenting: 1 part of all chunks; where phase 2
 * does not cut finer: the segments themselves.
 */
gdr_status_t gdr_forward_segment_parts(int variant, int B, int T, int H, int dv, int sms, int *parts,
                                       int *part_chunks);

/*
 * Synchronises `stream`, then reads and clears the library's device-side
 * error word.  Returns, since the previous call:
 *   GDR_ERR_TIMEOUT  a bounded wait inside a kernel (an mbarrier wait past its
 *                    limit of about a second) gave up; that kernel skipped its
 *                    remaining work and released its tensor memory;
 *   GDR_ERR_RANGE    a chunked-kernel operand left its range: an fp16 carry
 *                    operand (state, residual, W) above 6e4 in magnitude, or a
 *                    channel-wise decay spanning more than 2^120 within one
 *                    64-token chunk, or (backward) a reverse-carry operand
 *                    above 6e4; the results of that call are unreliable
 *                    and, for the forward, chunk=1 (per-token fp32) is the
 *                    safe path;
 *   GDR_ERR_CUDA     the synchronisation failed;
 *   GDR_OK           otherwise.
 */
gdr_status_t gdr_device_status(void *stream);

/* Human-readable name of a status, and the reason for the last rejected call. */
const char *gdr_status_string(gdr_status_t status);
const char *gdr_last_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
