/*
 * gdr.h -- C ABI of the B200 (sm_100a) gated delta-rule library.
 *
 * The library runs, per head, the gated delta-rule linear-attention recurrence
 *
 *   S_t = (I - k_t^T (b_t . k_t)) Diag(alpha_t) S_{t-1} + (w_t . k_t)^T v_t
 *   o_t = q_t S_t
 *
 * with row vectors q_t, k_t, alpha_t, b_t, w_t of length d_k, v_t and o_t of
 * length d_v, "." the elementwise product, and a d_k x d_v state S kept in
 * fp32. Sources for the operation:
 *   - write S <- S + k^T v and read o = q S, row vectors:
 *     "Recurrent Memory: Write, Erase, Decay, Read", section 01;
 *   - erase (delta rule, I - beta k^T k): same page, section 03, and
 *     "The Eraser Trilogy", "Eraser two";
 *   - decay Diag(alpha), scalar (Gated DeltaNet) or per channel (KDA), and the
 *     unified equation: same page, sections 04-05; "The Eraser Trilogy",
 *     "Eraser three";
 *   - channel-wise erase gate b and write gate w, collapsing to one scalar
 *     beta for KDA and Gated DeltaNet, decay absorbed into the erase factor:
 *     "Erase-then-Delta Attention" (Gated DeltaNet-2), abstract;
 *   - chunkwise-parallel evaluation: "Recurrent Memory", sections 03-04
 *     (reassociation into chunks; decay as a prefix sum of logs), and the
 *     chunkwise WY algorithm named in the Gated DeltaNet-2 abstract.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers: every array argument is a DEVICE pointer (memory the CUDA device
 *   can read/write). The caller owns every buffer; the library allocates no
 *   device memory, keeps no data between calls and never frees caller
 *   memory. The one CUDA object it keeps is described at
 *   gdr_chunk_fwd_workspace_size: an auxiliary stream and a few events per
 *   device, created by the first call that splits a general-form state pass
 *   into segments.
 * Layouts (contiguous, row-major, innermost last):
 *   q, k        [B, T, H, d_k]       chunk forward;  [B, H, d_k] decode
 *   v, o        [B, T, H, d_v]                       [B, H, d_v]
 *   scalar gate [B, T, H]                            [B, H]
 *   channel gate[B, T, H, d_k]                       [B, H, d_k]
 *   S0, S_T, S  [B, H, d_k, d_v] fp32
 * Element type: q, k, v, o and the gates all have type `dtype`
 *   (GDR_BF16 = bfloat16, GDR_FP32 = float). The state is always fp32 and
 *   all arithmetic accumulates in fp32.
 * Gates: alpha (decay) must lie in (0, 1]; b (erase) and w (write) are
 *   meant to lie in [0, 1] (not enforced). Kinds:
 *   GDR_GATE_NONE     the pointer must be NULL; alpha = 1, b = 0, w = 1.
 *   GDR_GATE_SCALAR   one value per token-head, used for every channel.
 *   GDR_GATE_CHANNEL  one value per token-head and key channel.
 *   GDR_GATE_TIED     w only: w := b (same values, pointer must be NULL);
 *                     b = w = beta is the KDA / Gated DeltaNet form.
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Calls are asynchronous: GDR_OK means the work was launched. Faults
 *   surface at the caller's next synchronisation.
 * Device status: `d_status`, if not NULL, is a device int the kernels OR
 *   GDR_DEVICE_* flags into (the caller zeroes it). Kernels never trap: every
 *   wait on the tensor-memory / TMA pipeline is bounded and, on expiry, sets
 *   GDR_DEVICE_TIMEOUT and ends the block cleanly.
 * Errors: argument problems are detected on the host before any launch and
 *   returned as gdr_status; nothing is launched in that case.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,   /* bad size, NULL where data is required, bad enum */
    GDR_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement */
    GDR_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    GDR_ERR_LAUNCH = 4,        /* the CUDA launch itself failed */
    GDR_ERR_NO_DEVICE = 5      /* no usable CUDA device / driver entry point */
} gdr_status;

/* Flags ORed into *d_status by the kernels. */
#define GDR_DEVICE_TIMEOUT 1       /* a bounded pipeline wait expired; results invalid */
#define GDR_DEVICE_DECAY_RANGE 2   /* a chunk took the exact fallback (see gdr_chunk_fwd); informational */

typedef enum { GDR_BF16 = 0, GDR_FP32 = 1 } gdr_dtype;

typedef enum {
    GDR_GATE_NONE = 0,
    GDR_GATE_SCALAR = 1,
    GDR_GATE_CHANNEL = 2,
    GDR_GATE_TIED = 3
} gdr_gate_kind;

/*
 * gdr_chunk_fwd -- forward pass over whole sequences (prefill / training
 * forward), evaluated chunk by chunk.
 *
 * Computes o_t for t = 0..T-1 of every (b, h) head, starting from S0 (or a
 * zero state when S0 is NULL), and writes the final state S_T when S_T is not
 * NULL. S_T may alias S0 (S0 is read once, before any write). o must not
 * alias any input.
 *
 * chunk: the chunk length of the chunkwise evaluation; 64 is the supported
 * value. The result does not depend on it beyond rounding.
 * Paths: dtype GDR_BF16 with d_k = 128 and d_v a multiple of 64 runs the
 * tcgen05 tensor-core chunk kernel (bf16 operands, fp32 accumulation, fp32
 * state on chip); so does d_k = 256 (the Gated DeltaNet head width of "How
 * Linear Attention Remembers", Table 1) with the Gated DeltaNet gates (scalar
 * alpha, scalar beta, w tied), d_v a multiple of 64 up to 256 and a
 * workspace. Every other supported shape (fp32, or 1 <= d_k <= 256 and
 * 1 <= d_v <= 1024 otherwise) runs an exact fp32 token-by-token CUDA kernel.
 * Decay: any alpha in (0, 1] is in range. With one decay per token (scalar
 * alpha) the tensor-core kernels form every ratio of decay products inside a
 * chunk per element, where it is at most 1. With channel-wise decay they
 * split each ratio into two factors around a per-chunk reference; a chunk
 * whose summed -log(alpha) in some channel exceeds about 160 cannot be split
 * that way, so that chunk alone is applied token by token in fp32 on CUDA
 * cores (exact, slower), and GDR_DEVICE_DECAY_RANGE is ORed into d_status to
 * say that the fallback ran.
 * Alignment: q, k, v, o and channel gates must be 16-byte aligned and, on
 * the tensor-core path, d_k and d_v rows 16-byte multiples (given by the
 * shape rules above).
 * workspace, workspace_bytes: optional caller-owned device scratch (NULL, 0
 * for none). When gdr_chunk_fwd_workspace_size() is non-zero for the call's
 * shape and gate form and workspace is not NULL, the forward runs in two
 * passes: first the per-chunk WY factors of every chunk of every head in
 * parallel (written to the workspace), then the state pass over the chunks.
 * Otherwise one kernel does both per chunk (at d_k = 256: the exact
 * kernel). Both give the same result up to rounding. The workspace must be 256-byte aligned and hold at least the
 * queried size; its contents on entry are ignored and on exit undefined.
 * Returns GDR_OK, GDR_ERR_INVALID_ARG (B, H < 1, T < 0, bad kinds, NULL
 * data, workspace smaller than required), GDR_ERR_UNSUPPORTED (chunk != 64,
 * shape beyond the limits above), GDR_ERR_MISALIGNED, GDR_ERR_LAUNCH or
 * GDR_ERR_NO_DEVICE. T = 0 writes S_T := S0 (or zeros) and launches nothing
 * else.
 */
gdr_status gdr_chunk_fwd(const void* q, const void* k, const void* v,
                         const void* alpha, const void* b, const void* w,
                         int alpha_kind, int b_kind, int w_kind,
                         const float* S0, void* o, float* S_T,
                         void* workspace, size_t workspace_bytes,
                         int B, int T, int H, int d_k, int d_v, int chunk,
                         int dtype, int* d_status, void* stream);

/*
 * gdr_chunk_fwd_grouped -- gdr_chunk_fwd with grouped query/key heads
 * ("How Linear Attention Remembers", Table 1: 16 q/k heads serving 32 value
 * heads). q and k are [B, T, H_qk, d_k]; v, o, the gates and the states have
 * H heads, and value head h reads q/k head h / (H / H_qk), so consecutive
 * value heads share one q/k head. Everything else is as gdr_chunk_fwd, which
 * is this call with H_qk = H; the workspace size does not depend on H_qk.
 * Returns GDR_ERR_INVALID_ARG also when H_qk < 1 or H is not a multiple of
 * H_qk.
 */
gdr_status gdr_chunk_fwd_grouped(const void* q, const void* k, const void* v,
                                 const void* alpha, const void* b, const void* w,
                                 int alpha_kind, int b_kind, int w_kind,
                                 const float* S0, void* o, float* S_T,
                                 void* workspace, size_t workspace_bytes,
                                 int B, int T, int H_qk, int H, int d_k, int d_v,
                                 int chunk, int dtype, int* d_status, void* stream);

/*
 * gdr_chunk_fwd_workspace_size -- bytes of scratch gdr_chunk_fwd's two-pass
 * path needs for this shape and gate form, or 0 when it has none. Two-pass
 * shapes: dtype GDR_BF16, T >= 1, and either d_k = 128, d_v in {64, 128}
 * with an erase gate (b_kind != GDR_GATE_NONE), or d_k = 256, d_v a multiple
 * of 64 up to 256 with the Gated DeltaNet gates. Sizes, in bytes, with
 * N = B*T*H:
 *   scalar alpha, tied scalar beta (Gated DeltaNet): 2 N (d_k + d_v + 64)
 *     (per-token rows of -W = -T Diag(beta g) K, of T Diag(beta) V and of
 *     the chunk's masked, decay-scaled q k^T block); at d_k = 256 also the
 *     rows of K~ = Diag(g_{n-1}/g) K: 2 N (2 d_k + d_v + 64);
 *   every other form: the per-token rows of -W 2^ref, q.g, k.g_{n-1}/g,
 *     the masked (q.rowf)(k.colf)^T block row and P (plus, with independent
 *     b and w, w.k.g_{n-1}/g and the masked (q.rowf)(w.k.colf)^T row), in
 *     bf16, g_{n-1} per chunk and channel in fp32, and one fp32 state
 *     [B, H, d_k, d_v] carried between the segments of a segmented state
 *     pass, each sub-buffer rounded up to 256 bytes.
 * With few (batch, head, 64-column) state tiles and long sequences the
 * general form splits the state pass into segments and runs the first pass of
 * later segments on an auxiliary stream while the state pass works through
 * earlier ones; the library then keeps that stream and a few events per
 * device for the rest of the process. Those are shared by every call on the
 * device: a call holds a per-device lock from its first event record to its
 * last stream wait, so concurrent calls from several host threads never wait
 * on each other's events. A call that finds the lock held by another thread,
 * or whose stream is being captured into a CUDA graph, does not split (it
 * launches one first pass and one state pass on its own stream), and so
 * neither touches the auxiliary stream nor serialises behind another caller.
 * Host-only; launches nothing.
 */
size_t gdr_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v,
                                    int alpha_kind, int b_kind, int w_kind,
                                    int dtype);

/*
 * gdr_chunk_fwd_static -- gdr_chunk_fwd without a caller workspace: the
 * two-pass path's scratch is a fixed device array inside the library
 * (gdr_chunk_fwd_static_capacity() bytes, one per device). The pages define
 * no such call; it exists so a caller can run the two-pass path while
 * allocating nothing.
 *
 * Arguments, layouts and results are those of gdr_chunk_fwd (which it calls
 * with that array as the workspace). Forms without a two-pass path use no
 * scratch. Returns GDR_ERR_UNSUPPORTED when the workspace the call needs
 * (gdr_chunk_fwd_workspace_size) exceeds the capacity, before touching the
 * device; otherwise as gdr_chunk_fwd.
 * Ownership and concurrency: the array is shared by every call on a device,
 * so calls whose executions overlap (different streams, threads or graphs
 * running concurrently) race on it and corrupt each other's results;
 * serialise them. The first call on each device looks the array up
 * (cudaGetSymbolAddress, which may load the module): make it before any
 * stream capture that records later calls. This call never splits the
 * general-form state pass into segments, so it creates no stream or event:
 * everything it launches goes to `stream`.
 */
gdr_status gdr_chunk_fwd_static(const void* q, const void* k, const void* v,
                                const void* alpha, const void* b, const void* w,
                                int alpha_kind, int b_kind, int w_kind,
                                const float* S0, void* o, float* S_T,
                                int B, int T, int H, int d_k, int d_v, int chunk,
                                int dtype, int* d_status, void* stream);

/* Bytes of the device array gdr_chunk_fwd_static uses (64 MiB). Host-only. */
size_t gdr_chunk_fwd_static_capacity(void);

/*
 * gdr_chunk_bwd -- backward pass of gdr_chunk_fwd: the gradients of a scalar
 * loss L with respect to every input, given dO = dL/do and dS_T = dL/dS_T.
 *
 * The pages call for a gate-aware backward pass that keeps training
 * parallel ("Erase-then-Delta Attention" (Gated DeltaNet-2), abstract) but
 * print no formula; the result is the exact derivative of the recurrence in
 * the file comment, taken in reverse token order with G = dL/dS_t
 * (e = b.k, u = w.k, S' = Diag(alpha_t) S_{t-1}, r_t = e S'):
 *   dq_t = dO_t S_t^T;  G += q_t^T dO_t;  dv_t = u G;  dr = -k G;
 *   dk_t = -G r_t^T + b.(S' dr^T) + w.(G v_t^T);
 *   db_t = k.(S' dr^T);  dw_t = k.(G v_t^T);
 *   dalpha_t = rowsum((G + e^T dr) . S_{t-1});  G <- Diag(alpha_t)(G + e^T dr);
 * and finally dS0 = G. Scalar gates get the sum over channels of the
 * per-channel gradient; with w tied to b, db holds the whole gradient of the
 * shared beta (both terms) and dw must be NULL.
 *
 * Inputs: q, k, v, alpha, b, w, kinds, S0 (NULL = zero state), dtype exactly
 *   as given to gdr_chunk_fwd; dO [B, T, H, d_v] in `dtype`; dS_T
 *   [B, H, d_k, d_v] fp32 or NULL (= 0).
 * Outputs, all fp32 and written completely (no accumulation into them):
 *   dq, dk [B, T, H, d_k]; dv [B, T, H, d_v]; dalpha, db, dw in the layout of
 *   their gate ([B, T, H] scalar, [B, T, H, d_k] channel), NULL exactly when
 *   the gate has no data of its own (kind NONE, or w TIED); dS0
 *   [B, H, d_k, d_v] or NULL (not written).
 * workspace: caller-owned device scratch of at least
 *   gdr_chunk_bwd_workspace_size() bytes, 256-byte aligned; contents on
 *   entry ignored, on exit undefined.
 * Method: the state gradient G follows its own backward recurrence
 *   G_{t-1} = Diag(alpha_t)(I - e^T k) G_t + q_{t-1}^T dO_{t-1}, which does
 *   not involve S, so the sequential work is two independent passes: forward
 *   (S at every 64-token chunk start, r_t) and backward (G at every chunk
 *   end, dr_t = -k G, dv_t, dS0). A chunk-parallel kernel then forms dq, dk
 *   and the gate gradients of each chunk from its start state, end
 *   gradient, r and dr:
 *   - the Gated DeltaNet form in bf16 with d_k = d_v = 128 (alpha and b
 *     scalar, w tied) runs on tensor cores throughout (bf16 operands, fp32
 *     accumulation) and scans nothing token by token: the forward two-pass
 *     kernels give S at every chunk start and U_t = beta_t v_t - r_t, both
 *     stored in bf16 (the chunk kernel uses them only as tensor-core
 *     operands and for one inner product per chunk); the backward recurrence
 *     of G taken a chunk at a time (per chunk, with Y_j = k_j G_j, T the
 *     forward's UT transform and Aq its masked q k^T block:
 *     (I + A)^T Y = Diag(g_{n-1}/g) K G_in + Aq^T dO and
 *     G_out = g_{n-1} G_in + (Diag(g) Q)^T dO - (Diag(beta g) K)^T Y) gives
 *     G at every chunk end and dr (bf16), dv and dS0 (a first pass over all
 *     chunks forms the chunk factors, a second walks the chunks in reverse); then
 *     the chunk gradients as masked, decay-scaled products, one CTA per
 *     (chunk, head) writing dalpha and db directly. Every gradient of this
 *     form carries bf16 operand rounding. The bounded waits of these kernels
 *     OR GDR_DEVICE_TIMEOUT into *d_status (if not NULL) and end the kernel,
 *     leaving the outputs undefined;
 *   - every other form and dtype: fp32 on CUDA cores: one kernel scans the
 *     tokens in both directions at once, one warp per 8 state columns; the
 *     chunk kernel works per block of state rows, rebuilding the chunk's
 *     states elementwise; a third kernel sums scalar gates' gradients over
 *     the key channels; d_status unused.
 *   Deterministic (no atomics) on both paths.
 * Supported: chunk = 64, 1 <= d_k <= 256, d_v a multiple of 8 up to 256,
 *   ceil(T / 64) <= 65535 and B * H <= 65535. Every pointer 16-byte
 *   aligned, except scalar gates and their gradients (element aligned).
 * Returns GDR_OK, GDR_ERR_INVALID_ARG (bad sizes or kinds, a NULL array that
 * is required, a gradient pointer that does not match its gate, workspace
 * missing or too small), GDR_ERR_UNSUPPORTED, GDR_ERR_MISALIGNED or
 * GDR_ERR_LAUNCH. T = 0 writes dS0 := dS_T (or zeros) and launches nothing
 * else.
 */
gdr_status gdr_chunk_bwd(const void* q, const void* k, const void* v,
                         const void* alpha, const void* b, const void* w,
                         int alpha_kind, int b_kind, int w_kind,
                         const float* S0, const void* dO, const float* dS_T,
                         float* dq, float* dk, float* dv,
                         float* dalpha, float* db, float* dw, float* dS0,
                         void* workspace, size_t workspace_bytes,
                         int B, int T, int H, int d_k, int d_v, int chunk,
                         int dtype, int* d_status, void* stream);

/*
 * gdr_chunk_bwd_grouped -- gdr_chunk_bwd with grouped query/key heads, as in
 * gdr_chunk_fwd_grouped: q, k and their gradients dq, dk are [B, T, H_qk,
 * d_k]; value head h reads q/k head h / (H / H_qk). dq and dk of a q/k head
 * are the sums over the value heads that share it (added in head order).
 * The workspace is gdr_chunk_bwd_grouped_workspace_size() bytes; everything
 * else is as gdr_chunk_bwd, which is this call with H_qk = H. Returns
 * GDR_ERR_INVALID_ARG also when H_qk < 1 or H is not a multiple of H_qk.
 */
gdr_status gdr_chunk_bwd_grouped(const void* q, const void* k, const void* v,
                                 const void* alpha, const void* b, const void* w,
                                 int alpha_kind, int b_kind, int w_kind,
                                 const float* S0, const void* dO, const float* dS_T,
                                 float* dq, float* dk, float* dv,
                                 float* dalpha, float* db, float* dw, float* dS0,
                                 void* workspace, size_t workspace_bytes,
                                 int B, int T, int H_qk, int H, int d_k, int d_v,
                                 int chunk, int dtype, int* d_status, void* stream);

/* Bytes of workspace gdr_chunk_bwd_grouped needs: gdr_chunk_bwd_workspace_size
 * plus, when H_qk < H, per-value-head dq and dk (2 x B T H d_k fp32, each
 * rounded up to 256 bytes). 0 for bad sizes. Host-only. */
size_t gdr_chunk_bwd_grouped_workspace_size(int B, int T, int H_qk, int H, int d_k, int d_v);

/* Bytes of workspace gdr_chunk_bwd needs (0 for T < 1 or bad sizes): fp32
 * chunk-start states and chunk-end state gradients (2 x B H ceil(T/64) d_k
 * d_v), r_t and dr_t of every token (2 x B T H d_v; the tensor-core form
 * keeps bf16 copies in the first half of each of these four regions), and scalar-gate partial
 * sums (3 x ceil(d_k / RB) x B T H, RB = 128 / (d_v / 8 rounded up to a power
 * of two)), and when d_k = d_v = 128 the forward's per-token -W, P and
 * q k^T block rows (B T H (d_k + d_v + 64) bf16; the gradient pass's
 * per-token rows of its chunk factors, B T H (128 + 64 + 128) bf16, reuse
 * that region), each rounded up to 256 bytes. Host-only; launches nothing. */
size_t gdr_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v);

/*
 * gdr_decode_step -- one token per head (autoregressive decoding).
 *
 * Applies one step of the recurrence to every (b, h) head: S is read and
 * overwritten in place with S_new, and o = q S_new is written. One pass over
 * S: the two column reductions (b.k.alpha) S and (q.alpha) S are taken while
 * S is read, and S_new is written from registers.
 * q, k [B, H, d_k]; v, o [B, H, d_v]; gates [B, H] or [B, H, d_k];
 * S [B, H, d_k, d_v] fp32. o must not alias S or the inputs.
 * Supported: 1 <= d_k <= 256, d_v in {16, 32, 64, 128, 256} (a head of
 * d_k > 128 and d_v = 256 runs as two blocks of 128 value columns: every
 * column's reductions over d_k stay inside its block).
 * Alignment: S, o, q, k, v and channel gates must be 16-byte aligned.
 * The step is a programmatic dependent launch on `stream`: its blocks may be
 * scheduled while the previous kernel on the stream finishes, and each waits
 * for that kernel's completion before reading anything, so stream order is
 * kept as for any launch.
 * Returns as gdr_chunk_fwd.
 */
gdr_status gdr_decode_step(const void* q, const void* k, const void* v,
                           const void* alpha, const void* b, const void* w,
                           int alpha_kind, int b_kind, int w_kind,
                           float* S, void* o, int B, int H, int d_k, int d_v,
                           int dtype, int* d_status, void* stream);

/*
 * gdr_decode_step_grouped -- gdr_decode_step with grouped query/key heads:
 * q, k are [B, H_qk, d_k], v, o, gates and S have H heads, value head h reads
 * q/k head h / (H / H_qk). gdr_decode_step is this call with H_qk = H.
 * Returns GDR_ERR_INVALID_ARG also when H_qk < 1 or H % H_qk != 0.
 */
gdr_status gdr_decode_step_grouped(const void* q, const void* k, const void* v,
                                   const void* alpha, const void* b, const void* w,
                                   int alpha_kind, int b_kind, int w_kind,
                                   float* S, void* o, int B, int H_qk, int H,
                                   int d_k, int d_v, int dtype, int* d_status,
                                   void* stream);

/*
 * gdr_selftest_bounded_wait -- diagnostic for the kernels' bounded waits.
 *
 * Launches one block that waits, with the bounded mbarrier wait used by the
 * tensor-core kernels (poll count and a 2 s %globaltimer limit), on a barrier
 * that nothing ever completes. The block gives up, ORs GDR_DEVICE_TIMEOUT
 * into *d_status (device int, required) and ends; the CUDA context stays
 * usable. Asynchronous on `stream`. Returns GDR_OK, GDR_ERR_INVALID_ARG
 * (NULL d_status) or GDR_ERR_LAUNCH. No page source defines this; it tests
 * the library's own failure handling.
 */
gdr_status gdr_selftest_bounded_wait(int* d_status, void* stream);

/* Human-readable name of a gdr_status value (static storage, never NULL). */
const char* gdr_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
