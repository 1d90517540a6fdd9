/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet token mixer forward pass
 * (chunked prefill and single-token decode) on NVIDIA B200 (sm_100a).
 *
 * The operation. For every sequence n and value head h the mixer carries a
 * state S (d_v x d_k, fp32) through the gated delta rule
 *
 *     q^_t = q_t / sqrt(|q_t|^2 + 1e-6) * scale,   k^_t = k_t / sqrt(|k_t|^2 + 1e-6)
 *     S_t  = alpha_t S_{t-1} (I - beta_t k^_t k^_t^T) + beta_t v_t k^_t^T,  alpha_t = exp(g_t)
 *     o_t  = S_t q^_t
 *
 * The Herbert pages name this recurrence as the Gated DeltaNet mixer of
 * Qwen3.5 ("On descend d'un cran", section "Ce que fait le moteur"; "On
 * descend d'un cran : #001 un compilateur pour moteur de LLM", section "Un
 * compilateur, pas une bibliothèque de kernels"), run it in two regimes --
 * the prompt in blocks at prefill, one row per token at decode -- and fuse
 * the whole decode step into one launch ("One level down: #004 the same
 * compiler on Apple's chips", section "Decode"). Their numerical contract is
 * bf16 activations with f32 accumulation and IEEE rounding, no fast-math
 * ("On descend d'un cran : #002 le même compilateur sur un GPU", section "Le
 * contrat numérique"; "One level down: #004", section "In short"). The
 * equation itself is not printed on the pages; the gated delta rule above is
 * the reading this library implements. States are fp32; gdn_decode_bf16_state
 * also offers the Metal article's bf16 state storage for decode.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers (cudaMalloc'd or equivalent),
 *     row-major with the innermost index last, contiguous, 16-byte aligned.
 *     The caller owns every buffer; the library never allocates, frees or
 *     synchronises (except gdn_device_error, which synchronises the stream).
 *   - dtype GDN_BF16: q, k, v, o are bf16 (o rounded to nearest even from
 *     fp32). GDN_F16: q, k, v, o are IEEE f16 (o rounded to nearest even),
 *     the pages' second numerical mode ("One level down: #004 the same
 *     compiler on Apple's chips", section "f16"); values beyond the f16
 *     range are the caller's concern. GDN_F32: q, k, v, o are fp32. g and
 *     beta are fp32 in every case, and so are the states, except in
 *     gdn_decode_bf16_state. Arithmetic is fp32 accumulation throughout.
 *   - Grouped heads: Hv must be a multiple of Hqk; value head h reads
 *     query/key head floor(h / (Hv / Hqk)) (contiguous groups).
 *   - g is the log-decay ln(alpha) (<= 0 in normal use); beta is used as given.
 *   - scale <= 0 selects d_k^-1/2.
 *   - stream is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued asynchronously; outputs are valid once the stream reaches it.
 *   - Errors: arguments are checked on the host before anything is enqueued;
 *     a failed check returns a status, enqueues nothing and writes nothing.
 *     A launch failure returns GDN_ERR_CUDA. gdn_last_error() returns a
 *     message for the calling thread's last failure.
 *   - Every device-side wait is bounded; a wait that runs out sets a device
 *     error word instead of spinning forever. gdn_device_error() reads it.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, bad cu_seqlens */
    GDN_ERR_UNSUPPORTED = 2,    /* valid but unsupported shape/dtype combination */
    GDN_ERR_CUDA = 3,           /* a CUDA call or launch failed */
    GDN_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait ran out (gdn_device_error) */
    GDN_ERR_DEVICE_CHECK = 5    /* an index check of the GDN_DEBUG build failed (gdn_device_error) */
} gdn_status;

typedef enum gdn_dtype {
    GDN_BF16 = 0,   /* bfloat16 */
    GDN_F32 = 1,    /* IEEE binary32 */
    GDN_F16 = 2     /* IEEE binary16 */
} gdn_dtype;

/*
 * Launch plan of the tensor-core prefill (bf16, dk = dv = 128). The kernel
 * splits its CTAs into ones that carry the recurrence state from chunk to
 * chunk, each owning a slice of `dvp` state rows of one (sequence, value head)
 * at a time, and ones that prepare the chunks' state-independent operands.
 * A field of 0 keeps the library's choice (a cost model of the two sides);
 * dvp must be 0, 32, 64 or 128 and n_chain_ctas >= 0. A requested plan is
 * clamped as gdn_prefill_plan documents. The result does not depend on the
 * plan beyond rounding.
 */
typedef struct gdn_plan {
    int dvp;            /* state rows per state-carrying CTA: 32, 64, 128 (0: the model's) */
    int n_chain_ctas;   /* number of state-carrying CTAs (0: the model's) */
} gdn_plan;

/* Library version, (major << 16) | minor. */
int gdn_version(void);

/*
 * Bytes of device workspace gdn_prefill needs for this problem: 0 unless the
 * tensor-core kernel runs it (GDN_BF16 or GDN_F16, dk = dv = 128). The tensor-core
 * kernel splits its CTAs into ones that prepare, per (value head, chunk), the
 * state-independent operands of the chunk and ones that carry the state from
 * chunk to chunk; the workspace holds the ring of prepared packages between
 * them (12 slots of 50 176 bytes per chain running at once, at most 74 chains)
 * and the ring's flags. It is at most about 44.6 MB however many sequences
 * there are. Depends only on the arguments given; a call zeroes the flags it
 * needs, so the contents on entry do not matter.
 */
size_t gdn_prefill_workspace_bytes(int n_seqs, int Hv, int dk, int dv, gdn_dtype dtype);

/*
 * The launch plan gdn_prefill_ex's tensor-core kernel would use for a problem
 * of n_seqs sequences, total_T tokens and Hv value heads on a device with
 * sm_count multiprocessors (0: the current device's), given the `requested`
 * plan (NULL: none): *dvp state rows per state-carrying CTA (32, 64 or 128),
 * *n_chain_ctas state-carrying CTAs (the other CTAs prepare packages) and the
 * *rounds in which the sequence-heads run. Clamping, as a launch applies it:
 * a requested dvp without a CTA count keeps the model's chains per round; the
 * count is capped at sm_count - 1, at the slices there are to run and at 74
 * chains at a time, and rounded down to whole chains (at least one).
 * Host only: touches no device memory and launches nothing (with sm_count > 0
 * it needs no GPU at all).
 * Returns GDN_ERR_UNSUPPORTED where the tensor-core kernel does not run
 * (GDN_F32, or dk, dv other than 128: those shapes run on the fp32 SIMT
 * kernel) and GDN_ERR_INVALID_ARG for a null output, an invalid
 * request, n_seqs or Hv <= 0, total_T < 0, or fewer than 16 multiprocessors.
 */
gdn_status gdn_prefill_plan(int n_seqs, int64_t total_T, int Hv, int dk, int dv, gdn_dtype dtype, int sm_count,
                            const gdn_plan *requested, int *dvp, int *n_chain_ctas, int *rounds);

/*
 * Chunked prefill over packed variable-length sequences.
 *
 *   q, k       [total_T, Hqk, dk]   dtype
 *   v          [total_T, Hv, dv]    dtype
 *   g, beta    [total_T, Hv]        fp32
 *   state_in   [n_seqs, Hv, dv, dk] fp32, or NULL for a zero initial state
 *   cu_seqlens [n_seqs + 1]         int32, DEVICE; cu_seqlens[0] = 0,
 *                                   non-decreasing, cu_seqlens[n_seqs] = total_T
 *   o          [total_T, Hv, dv]    dtype (output)
 *   state_out  [n_seqs, Hv, dv, dk] fp32 (output; may alias state_in exactly)
 *   workspace  device scratch of at least gdn_prefill_workspace_bytes(...)
 *              bytes (its contents on entry do not matter)
 *   chunk      tokens per chunk; 0 selects the default (64 for bf16 with
 *              dk = dv = 128, else 16). The result does not depend on it
 *              beyond rounding.
 *
 * Supported: GDN_BF16 or GDN_F16 with dk = dv = 128 and chunk 64
 * (tensor-core kernel: every tensor-core operand in the input's 16-bit
 * format, fp32 accumulation and state); GDN_F32 (and the 16-bit types with
 * other sizes or chunks) with dk, dv in {16, 32, 64, 128} and chunk in
 * {16, 32, 64} (fp32 SIMT kernel). total_T < 2^31. The
 * tensor-core kernel runs the sequence-heads in at most 1024 rounds of up to
 * 74 at a time; larger problems return GDN_ERR_UNSUPPORTED (split them
 * across calls). It is one cooperative launch with one CTA on every SM of the
 * device: other work on the device runs before or after it, not beside it.
 * How it splits the work (the width of the state slices and the number of
 * CTAs that carry states) is chosen from the problem's shape; gdn_prefill_ex
 * takes an explicit plan instead.
 * cu_seqlens is read on the device only; a cu_seqlens that breaks the rules
 * above is not detected on the host -- sequences with negative length are
 * treated as empty and tokens outside [0, total_T) are never read.
 */
gdn_status gdn_prefill(const void *q, const void *k, const void *v,
                       const float *g, const float *beta,
                       const float *state_in, const int32_t *cu_seqlens,
                       int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv,
                       float scale, int chunk, gdn_dtype dtype,
                       void *o, float *state_out,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_prefill with an explicit launch plan for the tensor-core kernel (see
 * gdn_plan; NULL or zero fields: the library's choice, so that
 * gdn_prefill(...) is gdn_prefill_ex(..., NULL, stream)). The plan is an
 * argument of the call, not process state: concurrent calls from several host
 * threads each run their own. Ignored by the fp32 SIMT kernel. An invalid plan
 * returns GDN_ERR_INVALID_ARG before anything is enqueued.
 */
gdn_status gdn_prefill_ex(const void *q, const void *k, const void *v,
                          const float *g, const float *beta,
                          const float *state_in, const int32_t *cu_seqlens,
                          int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv,
                          float scale, int chunk, gdn_dtype dtype,
                          void *o, float *state_out,
                          void *workspace, size_t workspace_bytes,
                          const gdn_plan *plan, void *stream);

/*
 * Allocation-free variant of gdn_prefill for callers that cannot provide
 * device scratch memory of their own: code running inside memory that an
 * inference runtime planned ahead of time, plugins whose host framework owns
 * every allocation, or real-time loops that must not call an allocator. The
 * Herbert pages have no counterpart to it; it exists for integration only.
 *
 * It runs the same tensor-core prefill as gdn_prefill, with the workspace
 * taken from a scratch array compiled into the library (45 MiB of device
 * memory, the largest workspace the kernel can ask for, held on every device
 * that loads the library until the process exits). It calls no allocator.
 * Arguments are those of gdn_prefill without the workspace; the caller still
 * passes every input and output.
 *
 *   Supported: GDN_BF16, dk = dv = 128, chunk 0 or 64 (anything else returns
 *   GDN_ERR_UNSUPPORTED); every problem size gdn_prefill accepts fits the
 *   array.
 *   The array's device address belongs to the CUDA context the library's
 *   module is loaded in. Every call made outside stream capture looks it up
 *   with cudaGetSymbolAddress (with the calling thread's device current) and
 *   caches it with that context's id; a call under stream capture uses the
 *   cached address, so make a first call outside capture in that context
 *   before capturing a stream into a CUDA graph (otherwise GDN_ERR_CUDA).
 *   A context that was destroyed and created again (cudaDeviceReset) is
 *   recognised by its new id.
 *   All calls share the one array and each call clears the part that must
 *   start at zero on its stream: calls whose kernels can overlap on the GPU
 *   (different streams or host threads) race and must be serialised by the
 *   caller.
 */
gdn_status gdn_prefill_noalloc(const void *q, const void *k, const void *v,
                               const float *g, const float *beta,
                               const float *state_in, const int32_t *cu_seqlens,
                               int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv,
                               float scale, int chunk, gdn_dtype dtype,
                               void *o, float *state_out, void *stream);

/*
 * One decode step for B independent sequences, one token each; the fused
 * step of "One level down: #004 the same compiler on Apple's chips",
 * section "Decode": L2-normalise q and k, decay, rank-1 delta update and
 * the o = S q readout in one launch that streams each state once.
 *
 *   q, k    [B, Hqk, dk]     dtype
 *   v       [B, Hv, dv]      dtype
 *   g, beta [B, Hv]          fp32
 *   state   [B, Hv, dv, dk]  fp32, updated in place
 *   o       [B, Hv, dv]      dtype (output)
 *
 * Supported: dk and dv in {16, 32, 64, 128}, any dtype.
 */
gdn_status gdn_decode(const void *q, const void *k, const void *v,
                      const float *g, const float *beta, float *state,
                      int B, int Hqk, int Hv, int dk, int dv,
                      float scale, gdn_dtype dtype, void *o, void *stream);

/*
 * Diagnostic for the failure path, not part of the computation (the pages
 * have no counterpart). Enqueues one tiny kernel that runs the prefill
 * kernel's two kinds of bounded wait -- on a flag in global memory and on a
 * shared-memory mbarrier -- on objects nothing ever signals, each for about
 * max_wait_us microseconds (1 .. 1000000; ~2 GHz assumed). Both waits run out,
 * record the timeout in the device error word and return; the kernel ends
 * normally and the CUDA context stays usable. A following gdn_device_error()
 * then reports GDN_ERR_DEVICE_TIMEOUT. Returns GDN_ERR_INVALID_ARG for an
 * out-of-range max_wait_us, GDN_ERR_CUDA if the launch fails.
 */
gdn_status gdn_wait_selftest(int max_wait_us, void *stream);

/*
 * gdn_decode with the state stored in bf16: the same step, computed in fp32,
 * on a state [B, Hv, dv, dk] of bf16 values that is read, updated and written
 * back rounded to nearest even -- the storage contract of "One level down:
 * #004 the same compiler on Apple's chips", section "In short" (recurrence
 * states in bf16, arithmetic in f32). It moves half the bytes of the fp32
 * state per step; each step's rounding adds up to half a bf16 ulp per state
 * element, so results drift from the fp32-state decode over many steps.
 * o is computed from the updated state before it is rounded. Arguments,
 * sizes and errors as gdn_decode; state is a DEVICE pointer to bf16 values.
 */
gdn_status gdn_decode_bf16_state(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta, void *state,
                                 int B, int Hqk, int Hv, int dk, int dv,
                                 float scale, gdn_dtype dtype, void *o, void *stream);

/* Message describing the calling thread's most recent failure ("" if none). */
const char *gdn_last_error(void);

/*
 * Synchronise `stream` and read, then clear, the device error word of the
 * current device. Returns GDN_ERR_DEVICE_CHECK if an index check of a
 * GDN_DEBUG build failed (the message names the check's source line),
 * GDN_ERR_DEVICE_TIMEOUT if a bounded wait ran out in any kernel since the
 * last call, GDN_ERR_CUDA if synchronisation failed, else GDN_OK. Meant for
 * tests and debugging; not needed in normal use.
 */
gdn_status gdn_device_error(void *stream);

/*
 * 1 if this library was built with GDN_DEBUG (libgdn_debug.so), else 0. The
 * debug build checks, on the device, the ring positions and slots, sequence
 * bounds, token and head coordinates and state offsets that the tensor-core
 * prefill computes before it uses them; a failed check records
 * GDN_ERR_DEVICE_CHECK in the device error word and stops that CTA's work
 * (the waits of the others are bounded), instead of reading or writing out
 * of bounds. It never traps. Diagnostic only: the checks cost time, and the
 * pages have no counterpart. Same ABI as the normal build otherwise.
 */
int gdn_debug_checks(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
