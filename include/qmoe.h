/*
 * qmoe.h - C ABI of libqmoe, the B200 (sm_100a) routed mixture-of-experts FFN
 * with 2-/4-bit block-quantised experts.
 *
 * Sources (web pages on the Strata engine; the method is defined by them and by
 * the workload definitions of this library's synthetic configurations):
 *   [P1] hexlives, "Commitment is a speedup" - one model whose 24,576 experts
 *        are consulted about ten per token; the decode GEMV is bandwidth-bound
 *        and a tensor-core variant lost on single-token shapes (fourth
 *        paragraph).
 *   [P3] pyshine, Strata source-tree tour - "Understanding the Architecture":
 *        48 captured layer graphs fed through fixed-address device buffers; a
 *        gate-weighted moe_combine summed on the device; expert buffers whose
 *        geometry disagrees get an error, never a read at wrong offsets;
 *        router_top10.cu routes each token to
 *        ten experts; batched prefill in chunks of up to 8,192 tokens.
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer unless its name ends in _host.
 *     The caller owns all memory; no call allocates or frees device memory.
 *   - Every device pointer must be 16-byte aligned, except route tables
 *     (idx int32 [T,k], gate fp32 [T,k]), which need 4-byte alignment.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as
 *     qmoe_stream_t; 0 = legacy default stream) and capturable into a CUDA
 *     graph, except where stated.
 *   - Host-side validation failures return an error code and launch nothing.
 *   - Device-detected faults (an expert index outside [0, E), a repeated expert
 *     within one token's route, a device wait that ran out of its time budget)
 *     are written to the caller's int32 *dev_status (first error wins; 0 = ok)
 *     and the kernel leaves without touching memory out of bounds. Read it with
 *     qmoe_read_status() after synchronising the stream.
 *   - No exception crosses this ABI.
 */
#ifndef QMOE_H_
#define QMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef struct CUstream_st *qmoe_stream_t; /* identical to cudaStream_t */

typedef enum {
  QMOE_OK = 0,
  QMOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, size out of range */
  QMOE_ERR_GEOMETRY = 2,      /* tensor shapes disagree with the expert handle */
  QMOE_ERR_UNSUPPORTED = 3,   /* valid request outside what the library supports */
  QMOE_ERR_WORKSPACE = 4,     /* workspace smaller than *_workspace_bytes() */
  QMOE_ERR_CUDA = 5,          /* a CUDA runtime call failed */
  QMOE_ERR_TIMEOUT = 6,       /* a device-side wait exceeded its budget */
  QMOE_ERR_DEVICE_STATUS = 7, /* invalid routed index seen on the device */
  QMOE_ERR_RANGE = 8          /* decode activations too large for the exact router sums:
                                 a 16-element slice's partial logit reached 2^19 */
} qmoe_status;

enum { QMOE_Q2 = 2, QMOE_Q4 = 4 };        /* block formats (bits per code) */
enum { QMOE_F32 = 0, QMOE_BF16 = 1 };     /* activation dtypes */
enum { QMOE_GATE_UP = 0, QMOE_DOWN = 1 }; /* packed matrix kinds */

/* One layer's experts, already packed by qmoe_pack().
 *   gate_up: E experts x {gate [I,H], up [I,H]}   (reduction axis H)
 *   down   : E experts x down [H,I]               (reduction axis I)
 * gate_up_bytes / down_bytes are the sizes of the two buffers; a handle whose
 * sizes differ from qmoe_packed_bytes() of its E/H/I/fmt is refused with
 * QMOE_ERR_GEOMETRY: the expert-source contract of [P3] "Understanding the
 * Architecture" turns a geometry mismatch into an error instead of reading
 * the wrong rows.
 * Geometry limits: H and I multiples of 128; E <= 1024. */
typedef struct {
  int E, H, I, fmt;
  const void *gate_up;
  const void *down;
  size_t gate_up_bytes;
  size_t down_bytes;
} qmoe_experts;

/* ---------------------------------------------------------------- format --
 * Self-defined block format: 32 consecutive weights along the reduction axis
 * share fp16 scale d and fp16 min m, w = d*q + m, q a 2-bit (Q2) or 4-bit (Q4)
 * code. (Strata loads third-party GGUF quant types - [P3] "How It Works" - whose
 * specifications are not part of the method; this format takes their place.)
 *
 * Canonical input layout for qmoe_pack, per expert matrix [rows, K]:
 *   codes  uint8  [E, rows, K*bits/8]: Q2 code j in byte j/4 bits 2*(j%4);
 *                                     Q4 code j in byte j/2, low nibble = even j
 *   scales uint16 [E, rows, K/32, 2]:  fp16 (d, m) per block
 * For QMOE_GATE_UP the caller passes gate and up separately (rows = I, K = H);
 * for QMOE_DOWN rows = H, K = I and the *_up pointers are NULL.
 *
 * Packed layout (this library's choice): 16-row tiles; inside a tile the codes
 * are arranged so that lane l of a warp loads 16 contiguous bytes holding its
 * tensor-core operand fragments, followed by the tile's (d, m) pairs.
 * qmoe_packed_bytes() equals the canonical size (8 (Q2) or 16 (Q4) code bytes
 * + 4 scale bytes per 32-weight block): packing adds no padding. */
size_t qmoe_packed_bytes(int fmt, int kind, int E, int H, int I);

/* Pack one layer's canonical matrices into dst (device, qmoe_packed_bytes()
 * bytes). Errors: INVALID_ARG for null pointers or dst_bytes too small,
 * UNSUPPORTED for H or I not multiples of 128 or fmt not Q2/Q4. */
qmoe_status qmoe_pack(int fmt, int kind, int E, int H, int I,
                      const uint8_t *codes_gate_or_down, const uint16_t *scales_gate_or_down,
                      const uint8_t *codes_up, const uint16_t *scales_up,
                      void *dst, size_t dst_bytes, qmoe_stream_t stream);

/* ---------------------------------------------------------------- router --
 * Router GEMV, softmax, top-k with renormalised gates ([P3] router_top10.cu,
 * "Understanding the Architecture"; ten experts per token in [P3]'s end-to-end
 * walk-through). For each token t:
 *   l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias[e])     accumulated in float64
 *   idx[t,:] = the k largest l[t,:], by value descending, ties to lower e
 *   gate[t,j] = exp(l[t,idx[t,j]] - l[t,idx[t,0]]) / sum_j' exp(...)
 * Inputs: Wr fp32 [E,H] row-major; bias fp32 [E] or NULL; x [T,H] fp32
 * (x_dtype QMOE_F32) or bf16 (QMOE_BF16). Outputs: idx int32 [T,k] and
 * gate fp32 [T,k]. Workspace: qmoe_route_workspace_bytes(T, E) bytes, zeroed
 * once before first use (it is left zeroed by every completed call).
 * Limits: 1 <= k <= 16, k <= E <= 1024, H multiple of 128, T >= 1; with fp32
 * x and T <= 8 also H <= 65,536.
 * T <= 8 with fp32 x runs the decode router: every 16-element slice partial
 * sum_h x*Wr is a float64 fused multiply-add chain, rounded to an integer in
 * units of 2^-32 and summed exactly, so the logit does not depend on how the
 * work is split (the fused layer stack forms the same logits); one warp per
 * token then selects from shared memory. A slice partial of magnitude 2^19 or
 * more sets QMOE_ERR_RANGE in the status word. Larger T or bf16 x runs the prefill router:
 * approximate logits on the integer tensor cores (16-bit fixed point in two
 * 8-bit limbs) with a proven error bound pick a few candidates per token,
 * whose float64 logits (exact products, float64 sums) decide the selection
 * and the gates. */
size_t qmoe_route_workspace_bytes(int T, int E);
qmoe_status qmoe_route(const float *Wr, const float *bias, const void *x, int x_dtype,
                       int T, int H, int E, int k, int32_t *idx, float *gate,
                       void *workspace, size_t workspace_bytes, int32_t *dev_status,
                       qmoe_stream_t stream);

/* Residual RMSNorm fused in front of the router (the gated residual stream
 * shared by all blocks, [P3] "Understanding the Architecture"):
 *   x_out[t,:] = z / sqrt(mean(z^2) + eps),  z = x_in[t,:] + y[t,:]
 * then routes x_out exactly like qmoe_route (fp32 activations, T <= 8).
 * x_out must not alias x_in or y. */
qmoe_status qmoe_residual_route(const float *x_in, const float *y, float eps, float *x_out,
                                const float *Wr, const float *bias, int T, int H, int E, int k,
                                int32_t *idx, float *gate, void *workspace,
                                size_t workspace_bytes, int32_t *dev_status,
                                qmoe_stream_t stream);

/* Standalone residual RMSNorm: x_out = RMSNorm(x_in + y), fp32 [T,H], with the
 * same arithmetic as the norm inside qmoe_residual_route (and the fused stack).
 * x_out may alias x_in. H a multiple of 16. */
qmoe_status qmoe_rmsnorm_residual(const float *x_in, const float *y, float eps, float *x_out,
                                  int T, int H, qmoe_stream_t stream);

/* ----------------------------------------------------- router, fixed scratch --
 * qmoe_route for callers that cannot allocate device memory for a workspace:
 * a host program that owns only its input and output buffers and has no
 * allocator, or a serving loop that may not call into one (an allocation can
 * synchronise the device). This entry point has no counterpart in the
 * method's sources; it is an interface convenience of this library.
 * It runs the same single-pass decode router as qmoe_route with fp32 x, with
 * its scratch (the exact integer partial-logit sums and a 256-byte completion
 * ticket) held in one fixed device array of QMOE_ROUTE_FIXED_SCRATCH_BYTES
 * bytes inside the library; nothing is allocated.
 * Limits: 1 <= T <= QMOE_ROUTE_FIXED_MAX_T, E <= QMOE_ROUTE_FIXED_MAX_E,
 * 1 <= k <= 16, H a multiple of 128 and at most 65,536; larger requests
 * return UNSUPPORTED.
 * The first call on each device looks up the array's address and zeroes it
 * synchronously (cudaGetSymbolAddress, cudaMemset; the ticket must start at
 * zero and every completed call leaves it at zero). Make that first call
 * before capturing any stream. Calls that may run at the same time on one
 * device (other streams, other host threads) share the array and race: keep
 * them on one stream. */
#define QMOE_ROUTE_FIXED_MAX_T 8
#define QMOE_ROUTE_FIXED_MAX_E 1024
#define QMOE_ROUTE_FIXED_SCRATCH_BYTES (QMOE_ROUTE_FIXED_MAX_T * QMOE_ROUTE_FIXED_MAX_E * 8 + 256)
qmoe_status qmoe_route_fixed(const float *Wr, const float *bias, const float *x, int T, int H, int E, int k,
                             int32_t *idx, float *gate, int32_t *dev_status, qmoe_stream_t stream);

/* -------------------------------------------------------------- decode FFN --
 * Routed expert FFN with the gate-weighted combine on the device ([P3]
 * moe_combine, native_moe.cu, "Understanding the Architecture"; [P1] the
 * bandwidth-bound decode GEMV), for decode and speculative-verify batches:
 *   for every token t and slot j, e = idx[t,j]:
 *     h = silu(Wg_e x_t) * (Wu_e x_t),  silu(a) = a / (1 + exp(-a))
 *   y[t,:] = sum_j gate[t,j] * (Wd_e h)        (summed in slot order)
 * x fp32 [T,H]; idx int32 [T,k]; gate fp32 [T,k]; y fp32 [T,H] (overwritten).
 * Limits: 1 <= T <= 8, 1 <= k <= 16. One cooperative grid of one CTA per SM:
 * weights stream through shared memory with bulk asynchronous copies and are
 * contracted on tensor cores (codes x activations in 24-bit fixed point per
 * 32-element block, held as three signed 8-bit limbs; exact integer block
 * sums, fp32 scaling per block).
 * Workspace: qmoe_decode_workspace_bytes(T, k, H, I), zeroed once before first
 * use (every completed call leaves its barrier words as it found them).
 * Errors: GEOMETRY if the handle's H/I/E do not match; device status for an
 * index outside [0, E) or a repeated expert in one token; TIMEOUT if a grid
 * barrier waited longer than its budget (about one second). */
size_t qmoe_decode_workspace_bytes(int T, int k, int H, int I);
qmoe_status qmoe_ffn_decode(const qmoe_experts *experts, const float *x, int T,
                            const int32_t *idx, const float *gate, int k, float *y,
                            void *workspace, size_t workspace_bytes, int32_t *dev_status,
                            qmoe_stream_t stream);

/* -------------------------------------------------------------- bucketing --
 * Token -> expert bucketing of a route (the routed pairs regrouped per expert
 * so each expert's weights are read once per chunk; [P3] batched prefill,
 * "Understanding the Architecture"). Pairs are numbered p = t*k + j. A stable
 * counting sort orders them by (expert, t, j):
 *   offsets int32 [E+1]: offsets[e] = number of pairs routed to experts < e
 *   perm    int32 [T*k]: perm[offsets[e] + i] = i-th pair (in pair order) of e
 *   active  int32 [E] or NULL: experts with at least one pair, ascending
 *   nactive int32 [1] or NULL: their count
 * Limits: E <= 1024, T*k <= 2^30. Two launches on `stream` over up to 148
 * CTAs (a per-CTA expert histogram, then placement); no CTA waits on another.
 * Workspace: qmoe_bucket_workspace_bytes(T, k, E) bytes, 16-byte aligned, no
 * initialisation needed. An index outside [0, E) sets the device status and
 * leaves offsets, perm, active and nactive unwritten. */
size_t qmoe_bucket_workspace_bytes(int T, int k, int E);
qmoe_status qmoe_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm,
                        int32_t *active, int32_t *nactive, void *workspace, size_t workspace_bytes,
                        int32_t *dev_status, qmoe_stream_t stream);

/* ------------------------------------------------------------- prefill FFN --
 * Routed expert FFN for prefill chunks of many tokens ([P3] batched prefill in
 * chunks of up to 8,192 tokens, "Understanding the Architecture"), computing
 * the same function as qmoe_ffn_decode on bf16 activations:
 *   y[t,:] = sum_j gate[t,j] * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  e = idx[t,j]
 * x bf16 [T,H]; idx int32 [T,k]; gate fp32 [T,k]; y fp32 [T,H] (overwritten).
 * Steps (all on `stream`): bucketing by expert, a tile plan, then two grouped
 * GEMMs on the tcgen05 tensor cores - bf16 operands (Q4 weights dequantised
 * to bf16 in shared memory, w = bf16(d)*q + bf16(m) rounded once), fp32
 * accumulation in tensor memory; the intermediate silu(g)*u is rounded to
 * bf16 between the two GEMMs. The second GEMM writes every routed pair's
 * gate-scaled output row (fp32, in bucket order) to the workspace, and a
 * combine kernel adds each token's k rows in slot order, so y is the same bit
 * for bit on every run. Measured relative error against the float64 oracle
 * at the 4096-token workload: about 8e-3 rel-RMS (bf16 operands), every token
 * row below 2e-2.
 * Limits: fmt Q4, H a multiple of 256, I a multiple of 128, k <= E <= 1024,
 * T*k <= 2^28. Workspace: qmoe_prefill_workspace_bytes(T, k, E, H, I) bytes
 * (T*k*H*4 of it for the pair rows), no initialisation needed. *dev_status
 * must be 0 on entry (a nonzero value skips the GEMMs); an index outside
 * [0, E) or an expert repeated within one token's route sets it. */
size_t qmoe_prefill_workspace_bytes(int T, int k, int E, int H, int I);
qmoe_status qmoe_ffn_prefill(const qmoe_experts *experts, const void *x, int T, const int32_t *idx,
                             const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                             int32_t *dev_status, qmoe_stream_t stream);
/* qmoe_ffn_prefill with kernel timing: events is a host array of three
 * cudaEvent_t (created by the caller, timing enabled) recorded on `stream`
 * right before the first grouped GEMM, between the two, and after the second
 * (before the combine); cudaEventElapsedTime of consecutive pairs gives the
 * two GEMM durations. flags: 0, or QMOE_PREFILL_ATOMIC_COMBINE for the
 * earlier combine (fp32 atomic additions straight into y from the second
 * GEMM; no combine kernel, run-to-run variation in y's last bits), kept to
 * measure one against the other. */
enum { QMOE_PREFILL_ATOMIC_COMBINE = 1 };
qmoe_status qmoe_ffn_prefill_timed(const qmoe_experts *experts, const void *x, int T, const int32_t *idx,
                                   const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                                   int32_t *dev_status, qmoe_stream_t stream, void *const *events, int flags);

/* ------------------------------------------------------------ layer stack --
 * L layers of route -> FFN -> residual RMSNorm captured once into one CUDA
 * graph ([P3] "Understanding the Architecture": 48 captured layer graphs; a
 * captured graph keeps the pointers it was recorded with, so each token's
 * values are written into buffers whose addresses never change).
 *   x_0 = input;  for l: (idx_l, gate_l) = route_l(x_l);  y_l = FFN_l(x_l);
 *                       x_{l+1} = RMSNorm(x_l + y_l)
 *   output = x_L
 * The descriptor's arrays are host arrays of L entries (copied at create).
 * The stack lives in caller workspace (qmoe_stack_workspace_bytes()); it keeps
 * the input, output and every layer's idx/gate there at fixed addresses. */
enum {
  QMOE_STACK_TIMING = 1,    /* capture CUDA events around every route and FFN node */
  QMOE_STACK_LAYERWISE = 2  /* use the per-layer kernel graph even where the fused kernel applies */
};
enum { QMOE_PATH_LAYERWISE = 0, QMOE_PATH_FUSED = 1 };

typedef struct {
  int L, T, k;
  float eps;
  const float *const *Wr;      /* L device pointers, fp32 [E,H] */
  const float *const *bias;    /* NULL or L device pointers (entries may be NULL) */
  const qmoe_experts *layers;  /* L handles with identical E/H/I; fmt may differ per layer */
  int flags;                   /* 0 or a combination of QMOE_STACK_TIMING, QMOE_STACK_LAYERWISE */
} qmoe_stack_desc;

typedef struct qmoe_stack qmoe_stack;

size_t qmoe_stack_workspace_bytes(const qmoe_stack_desc *desc);
/* Builds and instantiates the graph (host allocation of graph objects only).
 * Zeroes the workspace on `stream`. Not capturable. */
qmoe_status qmoe_stack_create(const qmoe_stack_desc *desc, void *workspace, size_t workspace_bytes,
                              qmoe_stream_t stream, qmoe_stack **out);
qmoe_status qmoe_stack_destroy(qmoe_stack *stack);
/* Fixed device buffers of the stack: input x [T,H], output x [T,H], idx [L,T,k],
 * gate [L,T,k] and the device status word. Any argument may be NULL. */
qmoe_status qmoe_stack_buffers(const qmoe_stack *stack, float **x_in, float **x_out,
                               int32_t **idx, float **gate, int32_t **dev_status);
/* Kernel launches in one replay of the stack's graph: 2L + 1 on the per-layer
 * path, 1 on the fused path. */
int qmoe_stack_kernels_per_replay(const qmoe_stack *stack);
/* Device address of the fused path's 32-bit grid-barrier counter inside the
 * stack's workspace (bit 31 flips once per grid barrier; it must read zero
 * between replays), or NULL on the per-layer path. For diagnostics and for
 * tests that make a barrier run out of its time budget: a counter preset to
 * 0x7FFFFFFF can never complete for some CTAs, so the replay ends with
 * QMOE_ERR_TIMEOUT after about one second instead of hanging. */
uint32_t *qmoe_stack_barrier_word(const qmoe_stack *stack);
/* Which path the stack runs. QMOE_PATH_FUSED (single-token stacks whose
 * geometry fits one SM's shared memory; a stack that mixes formats is laid
 * out for Q4 and takes each layer's format in turn): one persistent kernel runs all L
 * layers with two grid barriers per layer. QMOE_PATH_LAYERWISE:
 * qmoe_residual_route and qmoe_ffn_decode per layer, chained with
 * programmatic dependent launch. Both paths form a token's router logits from
 * the same integer sums of rounded 16-element slice partials (2^-32 units) and
 * give the same bits. */
int qmoe_stack_path(const qmoe_stack *stack);
/* Per-layer durations (ms) of the most recent completed replay of a
 * QMOE_STACK_TIMING stack: route_ms[l] spans layer l's router (with its fused
 * residual RMSNorm), ffn_ms[l] its FFN. Host arrays of L floats (either may be
 * NULL). Synchronous; UNSUPPORTED without the flag. Per-layer path: event
 * nodes around every kernel node. Fused path: the kernel's event-timed
 * duration split over the layers in proportion to each layer's median CTA
 * clock span; route_ms[l] is the part from the layer's start to its top-k. */
qmoe_status qmoe_stack_layer_times(const qmoe_stack *stack, float *route_ms, float *ffn_ms);
/* Raw phase stamps of the most recent replay of a QMOE_STACK_TIMING fused
 * stack: SM clock cycles (clock64 of each CTA's first consumer thread, so
 * compare only stamps of one CTA), int64 [L][*ctas][*points]: layer start,
 * top-k done, gate/up tiles start, gate/up tiles done, first grid barrier
 * passed, down tiles and router partials done, second grid barrier passed,
 * logits and normalised x ready (recorded between the first and second),
 * first gate/up tile landed (0 in a CTA without gate/up tiles), h limbs
 * landed, down tiles done, z written (these three 0 in CTAs that own no
 * output rows). count is the
 * capacity of cycles_host in entries (WORKSPACE if too small). UNSUPPORTED on the per-layer path or without the flag.
 * Synchronises the device. */
qmoe_status qmoe_stack_trace(const qmoe_stack *stack, int64_t *cycles_host, size_t count, int *ctas, int *points);
/* One graph replay on `stream`: reads the stack's input buffer, writes its
 * output buffer. */
qmoe_status qmoe_stack_decode(qmoe_stack *stack, qmoe_stream_t stream);
/* End to end from host memory: copies x_host (fp32 [T,H], ideally pinned) into
 * the input buffer, replays the graph and copies the output to x_out_host.
 * Asynchronous; synchronise `stream` before reading x_out_host. */
qmoe_status qmoe_stack_decode_host(qmoe_stack *stack, const float *x_host, float *x_out_host,
                                   qmoe_stream_t stream);

/* ------------------------------------------------------- n-gram row gather --
 * [P3] "Understanding the Architecture": besides the expert packs the model
 * keeps a large per-layer token-embedding table; a token's last three ids
 * are hashed into 16 row indices and only those rows are read. The pages fix
 * neither the hash nor the row format (a third-party 4-bit type), so both are
 * self-defined here, with SplitMix64's finaliser (Steele, Lea & Flood,
 * OOPSLA 2014) as the mixing function:
 *   mix64(z): z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
 *             z *= 0x94D049BB133111EB; z ^= z >> 31          (mod 2^64)
 *   G = 0x9E3779B97F4A7C15
 *   h = mix64(seed + G); then for each id of (a, b, c) in that order
 *       h = mix64(h ^ u), u = the id's 32-bit pattern zero-extended
 *   row i (i = 0..15) = floor(mix64(h + (i + 1) G) * R / 2^64)
 * Row format: the Q4 block format of this library in canonical layout, codes
 * uint8 [R][D/2] (code j of a row in byte j/2, low nibble for even j) and
 * scales uint16 [R][D/32][2] (fp16 d, m per 32-element block); w = d q + m,
 * exact in fp32.
 *
 * ngrams: device int32 [T][3], token t's ids (a, b, c) = (id_{t-2}, id_{t-1},
 *         id_t); any values (the caller pads the first positions).
 * out:    device fp32 [T][16][D]; out[t][i] = dequantised row i of token t.
 * rows:   device int32 [T][16] (the row indices), or NULL.
 * Limits: 1 <= R <= 2^31 - 1, D a multiple of 32 up to 8192, T >= 1.
 * Alignment: codes, out 16 bytes; ngrams, scales, rows 4 bytes.
 * Errors: INVALID_ARG (null or misaligned pointers, T < 1, R outside
 * [1, 2^31 - 1]), UNSUPPORTED (D outside the limits). Asynchronous on
 * `stream`. */
qmoe_status qmoe_ngram_gather(const int32_t *ngrams, int T, uint64_t seed, const uint8_t *codes,
                              const uint16_t *scales, int64_t R, int D, float *out, int32_t *rows,
                              qmoe_stream_t stream);

/* ------------------------------------------------------------------- misc -- */
/* Synchronous: copies *dev_status to the host and maps it to a status. */
qmoe_status qmoe_read_status(const int32_t *dev_status);
const char *qmoe_status_string(qmoe_status s);
/* Number of this library's kernel launches issued since load (host counter). */
uint64_t qmoe_launch_count(void);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif

#endif /* QMOE_H_ */
