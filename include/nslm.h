/*
 * nslm.h -- C ABI of libnslm, a B200 (sm_100a) library for SeedLM
 * seed-decompress matrix multiplies on routed mixture-of-experts layers.
 *
 * The method (sources, by page title and section):
 *  - "NanoSeedLM: LLM inference using pseudo-random numbers" (barnson.org),
 *    "Where this started": a weight matrix is cut into blocks of 8 weights;
 *    each block is a 16-bit LFSR seed, P tiny int4 coefficients and a shared
 *    exponent; running the LFSR from the seed gives an 8 x P basis U and the
 *    block is 2^e * U * c.  "What I changed: September 2026": the seed is the
 *    initial register state, and the weights are rebuilt inside the GPU
 *    kernels, in registers, every time (never decompressed to memory).
 *  - "K2-Horizon-MoVA-36B-A4B -- NanoSeedLM p4mx-q4v", "This upload": the
 *    tensors NAME.seeds (U16), NAME.coefs (U16), NAME.codes (U8) and
 *    NAME.exp_bias (I32); 100 routed FFN experts per layer, P = 4.
 *  - "Qwen3.8-Flash-Next-NanoSeedLM-P4", "The family": P = 4 costs 4.5 bits
 *    per weight, P = 3 costs 4.0 bits per weight.
 *
 * Definitions the pages leave open, fixed by this library:
 *  - LFSR: 16-bit Fibonacci register, polynomial x^16 + x^14 + x^13 + x^11 + 1;
 *    a step shifts right by one and enters s0^s2^s3^s5 at bit 15.
 *  - Basis: U[r][j] = (s_{1+8j+r} - 32768) / 32768, where s_0 is the seed and
 *    s_t the state after t steps; r = 0..7 (weight), j = 0..P-1 (coefficient).
 *  - Block: w_r = 2^(code + exp_bias[row]) * sum_j c_j U[r][j]; c_j is a
 *    two's-complement nibble in [-8, 7]; code an unsigned nibble in [0, 15].
 *    Every such weight is exactly representable in fp32.
 *  - Packed layout of an N x K matrix (nb = K / 8 blocks per row, row-major,
 *    little-endian), block b of row i covering W[i][8b .. 8b+7]:
 *      seeds    uint16 [N][nb]
 *      coefs    uint16 [N][nb]   c_j in bits 4j..4j+3; for P = 3 the exponent
 *                                code is in bits 12..15
 *      codes    uint8  [N][nb/2] P = 4 only: block 2m's code in the low
 *                                nibble of byte m, block 2m+1's in the high
 *                                nibble; NULL for P = 3
 *      exp_bias int32  [N]       must lie in [-100, 100]
 *
 * Conventions for every entry point:
 *  - Every pointer is a DEVICE pointer unless its comment says HOST.  The
 *    caller owns every buffer, the workspace included; the library never
 *    allocates, frees or synchronises.  All work is enqueued on `stream`
 *    (a cudaStream_t; NULL means the legacy default stream) and completes
 *    asynchronously.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns a negative status and launches nothing.  A launch
 *    failure returns NSLM_ERR_CUDA (the CUDA error is consumed).
 *  - Device arrays must be 16-byte aligned; K must be a multiple of 16 for
 *    P = 4 and of 8 for P = 3.
 *  - No function prints, aborts or throws.
 */
#ifndef NSLM_H
#define NSLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *nslm_stream_t;

/* Status codes. */
#define NSLM_OK 0
#define NSLM_ERR_ARG (-1)         /* null pointer, bad enum or count */
#define NSLM_ERR_ALIGN (-2)       /* a device pointer is not 16-byte aligned */
#define NSLM_ERR_SHAPE (-3)       /* N, K, P or a size outside what is supported */
#define NSLM_ERR_WORKSPACE (-4)   /* workspace missing or smaller than required */
#define NSLM_ERR_CUDA (-5)        /* a CUDA call or launch failed */
#define NSLM_ERR_TIMEOUT (-6)     /* a bounded device-side wait gave up; only
                                     nslm_device_status returns it, once the
                                     work it reports on has completed */
#define NSLM_ERR_UNSUPPORTED (-7) /* the current device is not sm_100 */

/* P = NSLM_P3C5: three coefficients of 5 bits ("NanoSeedLM: LLM inference
 * using pseudo-random numbers", "'Four bits is four bits'": P=3 with 5-bit
 * coefficients, 4.375 bits per weight).  Its 35 bits per block: the seeds
 * stream as usual; the coefs word holds c_0, c_1, c_2 as 5-bit two's
 * complement in bits 0-4, 5-9, 10-14 and bit 0 of the exponent code in bit 15;
 * codes: u8 [N][3 K / 64] holds code bits 1..3 of block b of a row at bits
 * 3b .. 3b+2 of the row's bit string, least significant bit first.  K must be
 * a multiple of 64.  Taken by nslm_seed_gemv, the debug decompression, the
 * decode FFN and layer stack (T <= 8, persistent and per-layer kernels), the
 * tensor-core FFN path (T > 8) and nslm_seed_grouped_gemm; the search, expert
 * cache, nibbles and hybrid entry points return NSLM_ERR_SHAPE for it. */
#define NSLM_P3C5 35

/* One packed seed matrix (see the layout above).  For a stack of E experts,
 * N = E * rows and expert e owns rows [e * rows, (e + 1) * rows). */
typedef struct {
    const uint16_t *seeds;
    const uint16_t *coefs;
    const uint8_t *codes;    /* NULL when P == 3 */
    const int32_t *exp_bias;
    int32_t N;
    int32_t K;
    int32_t P;               /* 3, 4 or NSLM_P3C5 */
} nslm_seed_matrix;

/* One MoE layer: gate and up are [E * inter][hidden], down is [E * hidden][inter]. */
typedef struct {
    nslm_seed_matrix gate;
    nslm_seed_matrix up;
    nslm_seed_matrix down;
} nslm_moe_layer;

/* Workspace sizing: op codes for nslm_workspace_bytes. */
#define NSLM_OP_GEMV 0
#define NSLM_OP_GROUPED_GEMM 1
#define NSLM_OP_MOE_FFN 2
#define NSLM_OP_MOE_STACK 3
#define NSLM_OP_MOE_FFN_HYBRID 4  /* E = E3 + E4 */

/* Bytes of workspace an operation needs (0 if none).  T = tokens, E =
 * experts, hidden/inter = FFN sizes, k = experts per token, L = layers (only
 * NSLM_OP_MOE_STACK uses L; pass 0 otherwise).  Host-only, never fails. */
size_t nslm_workspace_bytes(int32_t op, int32_t T, int32_t E, int32_t hidden,
                            int32_t inter, int32_t k, int32_t L);

/* Seed GEMV, the decode matrix-vector product ("Where this started": the
 * weights are regenerated from the seeds inside the multiply).
 *   y[m][i] = sum_k W[i][k] * x[m][k],  m < M, i < N.
 * x: bf16 bit patterns [M][K]; y: fp32 [M][N]; 1 <= M <= 8.
 * Accumulates in fp32; results match the fp64 product to about 1e-6
 * relative.  Uses no workspace (ws may be NULL). */
int32_t nslm_seed_gemv(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M,
                       float *y, void *ws, size_t ws_bytes, nslm_stream_t stream);

/* nslm_seed_gemv with flags (0 gives nslm_seed_gemv exactly):
 *   NSLM_GEMV_FIELDS_READY  the caller declares that no kernel enqueued
 *     earlier on `stream` writes W's seeds, coefs, codes or exp_bias.  The
 *     product kernel is launched with programmatic dependent launch in both
 *     forms and waits for its predecessor before it reads x or writes y; with
 *     this flag its first weight-field copies are issued before that wait, so
 *     they overlap the tail of the preceding kernel (e.g. the previous GEMV of
 *     a decode step).  If the declaration is false the result is undefined.
 *     It affects M = 1 with K % 64 == 0 (the one-vector kernel); other
 *     shapes run as without it.
 * Other bits return NSLM_ERR_ARG. */
#define NSLM_GEMV_FIELDS_READY 1u
int32_t nslm_seed_gemv_flags(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M,
                             float *y, uint32_t flags, nslm_stream_t stream);

/* Grouped seed GEMM over stacked experts, the batched (prefill) product of
 * "Qwen3.8-Flash-Next" prompt processing ("The prompt time ... the grouped
 * expert GEMMs", NanoSeedLM documentation index, Results).
 *   For every expert e and every row t in [offsets[e], offsets[e+1]):
 *     y[t][i] = sum_k W_e[i][k] * x[t][k],  i < rows = W->N / E.
 * x: bf16 [R][K], rows grouped by expert; offsets: int32 [E + 1] (DEVICE),
 * non-decreasing, offsets[0] = 0, offsets[E] = R; y: fp32 [R][rows].
 * Weights are regenerated into bf16 (round to nearest even) tiles and
 * multiplied on the tensor cores (tcgen05) with fp32 accumulation.  Requires
 * K % 64 == 0 and 1 <= E <= 1024; rows outside [0, R) are never read.  A
 * tensor-core wait that does not complete within about two seconds stops the
 * kernel and sets the first int32 of the workspace to 1 (0 otherwise).
 * Workspace: nslm_workspace_bytes(NSLM_OP_GROUPED_GEMM, R, E, K, rows, 1, 0). */
int32_t nslm_seed_grouped_gemm(const nslm_seed_matrix *W, int32_t E, const uint16_t *x_bf16,
                               const int32_t *offsets, int32_t R, float *y, void *ws,
                               size_t ws_bytes, nslm_stream_t stream);

/* Router: for each token, the k largest of E logits (descending; ties go to
 * the lower expert id) and the softmax of the k selected logits.
 * logits: fp32 [T][E]; ids: int32 [T][k]; w: fp32 [T][k]; 1 <= k <= 8,
 * k <= E <= 1024.  ("Why K2-Horizon-MoVA": 100 routed experts, top 8.) */
int32_t nslm_moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k,
                            int32_t *ids, float *w, nslm_stream_t stream);

/* Routed expert FFN for T tokens ("Why K2-Horizon-MoVA": routed FFN experts,
 * top 8; gate and up projections, SiLU, down projection):
 *   y[t] = sum_q w[t][q] * Down_e( SiLU(Gate_e x[t]) * (Up_e x[t]) ),  e = ids[t][q]
 * with SiLU(g) = g / (1 + exp(-g)).  gate/up: [E * inter][hidden];
 * down: [E * hidden][inter], all with the same P.  x: bf16 [T][hidden];
 * ids: int32 [T][k] in [0, E); w: fp32 [T][k]; y: fp32 [T][hidden].
 * T <= 8 runs the decode path (fp32 weights and hidden activations);
 * larger T runs the tensor-core path (bf16 weights, bf16 hidden activation;
 * hidden and inter multiples of 64, E <= 1024).  The first int32 of the
 * workspace is set nonzero if a device-side wait (the tensor-core pipeline,
 * or the grid barrier of a persistent decode kernel) gave up.
 * Workspace: nslm_workspace_bytes(NSLM_OP_MOE_FFN, T, E, hidden, inter, k, 0). */
int32_t nslm_moe_seed_ffn(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                          const nslm_seed_matrix *down, int32_t E, const uint16_t *x_bf16,
                          const int32_t *ids, const float *w, int32_t T, int32_t k, float *y,
                          void *ws, size_t ws_bytes, nslm_stream_t stream);

/* A routed expert FFN whose experts are packed with different P ("NanoSeedLM:
 * LLM inference using pseudo-random numbers", news list: hybrid P3 / P4 seed
 * packs, ~4.17 bits per weight; reading: each expert is P = 3 or P = 4 as a
 * whole).  p3: HOST pointer to the layer's E3 P = 3 experts (stacked as for
 * nslm_moe_seed_ffn); p4: its E4 P = 4 experts, same hidden and inter.  Expert
 * id e < E3 is p3's expert e, E3 <= e < E3 + E4 is p4's expert e - E3; other
 * ids contribute nothing.  y = the layer's output, as nslm_moe_seed_ffn
 * computes it over all E3 + E4 experts: the routed FFN runs per stack (the
 * same kernels, the same T-dependent path) and the two partial outputs are
 * added in a fixed order.  Workspace: nslm_workspace_bytes(
 * NSLM_OP_MOE_FFN_HYBRID, T, E3 + E4, hidden, inter, k, 0).  Launches: the
 * two FFNs' plus two. */
int32_t nslm_moe_seed_ffn_hybrid(const nslm_moe_layer *p3, int32_t E3, const nslm_moe_layer *p4,
                                 int32_t E4, const uint16_t *x_bf16, const int32_t *ids, const float *w,
                                 int32_t T, int32_t k, float *y, void *ws, size_t ws_bytes,
                                 nslm_stream_t stream);

/* The decode path of nslm_moe_seed_ffn (T <= 8) for callers that may not
 * allocate device memory: the scratch it needs lives in a 1 MiB array built
 * into the library (one per GPU that loads it, kept until the process exits),
 * so no workspace is passed and nothing is allocated.  The pages have no
 * counterpart; this is an interface convenience, not part of the method.
 *
 * Which callers this is for: code embedded in a host application whose
 * allocator owns the GPU's memory, latency-critical loops that cannot take an
 * allocation's implicit synchronisation, and callers that only receive input
 * and output pointers.
 *
 * Arguments, layout and results are those of nslm_moe_seed_ffn without ws and
 * ws_bytes.  Returns NSLM_ERR_WORKSPACE if the problem's workspace
 * (nslm_workspace_bytes(NSLM_OP_MOE_FFN, T, E, hidden, inter, k, 0)) exceeds
 * 1 MiB; T > 8 returns NSLM_ERR_SHAPE.
 * The first call on a device, made with that device current, looks up the
 * array's device address (cudaGetSymbolAddress) and caches it; make that first
 * call before capturing any stream.  All calls share the one array: calls
 * whose work overlaps on the GPU (e.g. on two streams at once) race and give
 * wrong results.  Each call rewrites what it reads, so the contents left by an
 * earlier call do no harm.  A grid-barrier wait that gives up (about 1 s) is
 * reported by nslm_device_status(NULL, stream), not by the return value.
 * The cached address belongs to the CUDA context it was looked up in: after
 * cudaDeviceReset the library must be reloaded before this entry point is
 * called again on that device. */
int32_t nslm_moe_seed_ffn_static(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                                 const nslm_seed_matrix *down, int32_t E, const uint16_t *x_bf16,
                                 const int32_t *ids, const float *w, int32_t T, int32_t k,
                                 float *y, nslm_stream_t stream);

/* A stack of L MoE layers for T <= 8 decode tokens.  Layer l routes with
 * logits[l] (fp32 [L][T][E]) and runs nslm_moe_seed_ffn on its input; the
 * next layer's input is bf16(y / sqrt(mean(y^2) + 1e-6)) per token (the pages
 * put attention between MoE layers; this normalisation stands in for it).
 * layers: HOST array of L layers (device pointers inside), all with the same
 * E, hidden, inter and P.  x0: bf16 [T][hidden]; y: fp32 [T][hidden], the
 * last layer's output.  Where the shape allows (T = 1, or T >= 2 with
 * hidden and inter multiples of 64) all layers run in one cooperative launch
 * per 64 layers after one routing launch; otherwise each layer takes two
 * launches.  The first int32 of the workspace is set nonzero if a grid
 * barrier wait of the persistent kernel gave up (about 1 s).
 * Workspace: nslm_workspace_bytes(NSLM_OP_MOE_STACK, T, E, hidden, inter, k, L). */
int32_t nslm_moe_stack_decode(const nslm_moe_layer *layers, int32_t L, int32_t E, int32_t k,
                              const float *logits, const uint16_t *x0_bf16, int32_t T,
                              float *y, void *ws, size_t ws_bytes, nslm_stream_t stream);

/* Seed search, the encoder ("NanoSeedLM: LLM inference using pseudo-random
 * numbers", "What I changed: September 2026": every block walks all 65,535
 * seeds; "'GPU search == CPU search'": the GPU search gives the C reference's
 * answer bit for bit).  For each block of 8 weights of w (fp32 [N][K], row
 * major, device) and every seed in [seed_lo, seed_hi] (1 <= seed_lo <=
 * seed_hi <= 65535) and code in 0..15:
 *   c = round_half_even(pinv(U(seed)) w_block / 2^(code + exp_bias[row])),
 *       clamped to [-8, 7];  pinv(U) = (U^T U)^-1 U^T by Gauss-Jordan
 *       elimination with partial pivoting, fp64, no fused multiply-add
 *   err = sum_r (w_r - 2^(code + exp_bias[row]) (U c)_r)^2, fp64
 * The smallest err wins; ties go to the larger code, then the lower seed.
 * imp: fp32 [K] per-column importances (the mean square of each column's
 * input activation, "Qwen3.8-Flash-Next-NanoSeedLM-P4", "How it works"), or
 * null.  With imp, d_r = imp[8 b + r] weights each term of err, and the fit is
 * the weighted least-squares one: pinv = (U^T D U)^-1 U^T D with
 * A[a][b] = sum_r ((U_ra U_rb) d_r) and B[a][r] = U_ra d_r, then
 * err = sum_r d_r ((w_r - ...)^2); unit importances give the unweighted
 * answer.  Importances should be finite and >= 0 (they are not checked);
 * a block whose importances make every seed singular is unencodable.
 * out: the packed matrix to fill (N, K, P give the shape; K % 8 == 0, P=4
 * needs K % 16 == 0): seeds, coefs (and codes for P = 4) are WRITTEN;
 * exp_bias [N] is READ (the row biases to encode with).  err: fp64 [N][K/8]
 * of the winning errors, or null.  A block whose every seed is singular gets
 * seed 0, zero coefficients and err = +inf.  All pointers are device
 * pointers; the seed streams of out must not overlap w. */
int32_t nslm_seed_search(const float *w, const float *imp, const nslm_seed_matrix *out,
                         int32_t seed_lo, int32_t seed_hi, double *err, nslm_stream_t stream);

/* Routed experts in host memory behind a VRAM cache of recently used experts
 * ("NanoSeedLM" README, "Highlights": the CUDA engine can keep the routed
 * experts in RAM while a VRAM cache holds the recently used ones; LRU was the
 * pages' best policy).  One call prepares one layer's decode step:
 *   - a one-CTA kernel runs LRU over the routed pairs ids [T][k] (device, in
 *     order): a hit refreshes the slot; a miss takes the least recently used
 *     slot not used in this step (empty slots first, then the oldest, ties to
 *     the lower slot) and schedules a copy; slot_ids [T][k] (device) gets the
 *     slot of every pair (-1 for ids outside [0, E));
 *   - a copy kernel moves each missed expert's gate, up and down fields from
 *     the source stacks into its slot.
 * Then nslm_moe_seed_ffn(gate_cache, up_cache, down_cache, S, x, slot_ids, w,
 * ...) computes the layer.  No host synchronisation; graph-capturable.
 * *_src: the layer's E experts stacked as for nslm_moe_seed_ffn, in memory the
 * device can read: device memory, or pinned host memory (cudaHostAlloc /
 * cudaHostRegister) under unified addressing.  *_cache: S expert slots
 * stacked the same way, device memory, same hidden / inter / P.  Cache keys
 * are (layer, expert), so one cache can serve every layer of a stack.
 * state: device, nslm_expert_cache_state_bytes(S) bytes, zero-filled before
 * first use (an empty cache); int32 [0] calls so far, [1] copies of the last
 * call, [2] total hits, [3] total misses.  Needs T * k <= S <= 4096,
 * T * k <= 64, hidden and inter multiples of 64, 16-byte aligned streams.
 * Two launches. */
size_t nslm_expert_cache_state_bytes(int32_t slots);
int32_t nslm_expert_cache_fetch(const nslm_seed_matrix *gate_src, const nslm_seed_matrix *up_src,
                                const nslm_seed_matrix *down_src, int32_t E, int32_t layer,
                                const nslm_seed_matrix *gate_cache, const nslm_seed_matrix *up_cache,
                                const nslm_seed_matrix *down_cache, int32_t S, void *state,
                                const int32_t *ids, int32_t T, int32_t k, int32_t *slot_ids,
                                nslm_stream_t stream);

/* The "nibbles" layout of seed packs ("Qwen3.8-Flash-Next-NanoSeedLM-P4",
 * "Files": routed experts as NAME.seeds, NAME.nibbles and NAME.exp_bias).
 * nibbles: u8 [N][(P+1) * K / 16], device; block b of a row holds nibbles
 * (P+1)b .. (P+1)b+P, namely c_0 .. c_{P-1} (two's complement) and then the
 * exponent code, nibble n in byte n / 2 (low half for even n).  Seeds and
 * exp_bias are the same streams in both layouts.
 * nslm_unpack_nibbles WRITES out->coefs (and out->codes for P = 4) from the
 * nibbles (out->seeds and out->exp_bias are not touched);
 * nslm_pack_nibbles READS in->coefs (and in->codes) and WRITES nibbles.
 * For P = 3 the two layouts are the same bytes.  Shapes as for any matrix
 * (K % 8 == 0; P = 4: K % 16 == 0 and codes present).  One launch; buffers
 * must not overlap. */
int32_t nslm_unpack_nibbles(const uint8_t *nibbles, const nslm_seed_matrix *out, nslm_stream_t stream);
int32_t nslm_pack_nibbles(const nslm_seed_matrix *in, uint8_t *nibbles, nslm_stream_t stream);

/* Test export: the bounded device waits give up and report, they do not
 * hang.  kind 0: the grid-barrier wait of the persistent decode kernels,
 * waiting for one arrival on out[0..3] (status, arrivals, abort, as at the
 * head of the decode workspace; the caller initialises them: arrivals 0 makes
 * the wait run out, 1 lets it pass); on giving up it sets out[0] = 1 and
 * out[2] = 1.  out[4] = 1 if the wait passed, 0 if it gave up.
 * kind 1 / 2: the mbarrier wait of the tensor-core pipeline on a barrier
 * whose phase nothing completes (1) or that one arrival completed first (2);
 * out[0] = 1 if it passed, 0 if it gave up.  kind 3: the wait of the
 * one-token stack on a tagged 64-bit word (fp32 bits low, layer tag high),
 * here the word at out[6..7] (caller-initialised, out 8-byte aligned) waited
 * on for tag 1, with out[0..3] as the status words of kind 0; out[4] = 1 if it
 * passed, 0 if it gave up (then out[0] = 1, out[2] = 1); out[5] = the value
 * bits it saw.  cycles: the wait limit in SM clocks (> 0).  out: device, 5
 * int32 (8 for kind 3).  One launch of one CTA. */
int32_t nslm_debug_wait_probe(int32_t kind, int32_t *out, int64_t cycles, nslm_stream_t stream);

/* Test export: the bf16 hidden activations h = SiLU(gate x) * (up x) that the
 * last nslm_moe_seed_ffn call with T > 8 (the tensor-core path) left in its
 * workspace ws (ws_bytes, T, E, hidden, inter, k as in that call), written
 * to h_out [T * k][inter] (bf16 bit patterns, DEVICE) in pair order: row
 * t * k + q is token t's q-th routed expert.  Rows of pairs whose expert id was
 * outside [0, E) are not written.  It lets a test take the kernel's own
 * rounding of h to bf16 as given when it checks the down projection.  One
 * launch; T <= 8 returns NSLM_ERR_SHAPE (the decode path keeps h in fp32). */
int32_t nslm_debug_batched_hidden(const void *ws, size_t ws_bytes, int32_t T, int32_t E,
                                  int32_t hidden, int32_t inter, int32_t k, uint16_t *h_out,
                                  nslm_stream_t stream);

/* Test exports of the bounds-check build (libnslm built with
 * -DNSLM_BOUNDS_CHECK=1: python -m lfsr_seeded_moe_b200.build --bounds-check).
 * There every checked global access of the kernels compares its index with
 * the extent it was given; an index outside records a site number (1-2 field
 * copies by offset, 3-4 field loads by row, 5-6 the tensor-core producer's
 * field and token-row loads, 7-9 the tensor-core epilogue's stores, 10 the
 * decode kernels' h stores) and the access is skipped, so nothing traps.
 * nslm_debug_bounds_status waits for the device, then returns the first site
 * recorded since the previous call (0: none) and clears it.
 * nslm_debug_bounds_probe(W) launches one field copy one chunk past the end
 * of W (P = 4, K % 64 == 0, N >= 1), which its check refuses as site 1.  In
 * the normal build both return NSLM_ERR_UNSUPPORTED and launch nothing. */
int32_t nslm_debug_bounds_status(void);
int32_t nslm_debug_bounds_probe(const nslm_seed_matrix *W, nslm_stream_t stream);

/* Test export of the trace build of the library (-DNSLM_STACK1_TRACE=1:
 * python -m lfsr_seeded_moe_b200.build --trace).  There the one-token
 * persistent decode kernel (nslm_moe_stack_decode and nslm_moe_seed_ffn at
 * T = 1) stamps the device's global nanosecond timer at the phase boundaries
 * of every layer: stamp k of CTA c at layer l of a launch is out[(k * 256 +
 * c) * 64 + l] (k: 0 layer start, 1 input x staged, 2 the CTA's gate/up phase
 * done, 3 past the grid barrier, 5 h staged, 6 thread 0's down tasks done,
 * 4 the CTA's down phase done; CTAs below 256, layers below 64 of the last
 * launch).  out: HOST, n_words >= 8 * 256 * 64 uint64.  Synchronises the
 * device.  In the normal build returns NSLM_ERR_UNSUPPORTED. */
int32_t nslm_debug_stack_trace(uint64_t *out, size_t n_words);

/* Test exports: the regenerated weights themselves, written out densely.
 * w_out: fp32 [N][K] (exact) or bf16 bit patterns [N][K] (round to nearest
 * even of the exact value).  Not on the hot path. */
int32_t nslm_debug_decompress(const nslm_seed_matrix *W, float *w_out, nslm_stream_t stream);
int32_t nslm_debug_decompress_bf16(const nslm_seed_matrix *W, uint16_t *w_out,
                                   nslm_stream_t stream);

/* Device-side status of the calls that used workspace ws: NSLM_OK, or
 * NSLM_ERR_TIMEOUT if a bounded wait of one of them gave up (the grid barrier
 * of a persistent decode kernel, about 1 s, or a tensor-core pipeline wait,
 * about 2 s).  Such a call has returned NSLM_OK to its caller, because the
 * wait happens on the GPU after the call returned; its output is then
 * incomplete.  The status is the first int32 of the workspace, which every
 * decode or tensor-core call rewrites at its start, so it reports the last
 * call that used ws.  ws = NULL reads the status of the built-in scratch of
 * nslm_moe_seed_ffn_static instead.
 * Not for the hot path: it waits for `stream` to finish (cudaStreamSynchronize)
 * and then copies the 4-byte word to the host, so it cannot be captured in a
 * CUDA graph.  Returns NSLM_ERR_CUDA if the stream reports an error. */
int32_t nslm_device_status(const void *ws, nslm_stream_t stream);

/* A static, human-readable name for a status code. */
const char *nslm_status_string(int32_t status);

/* Number of kernel launches the last successful call on this host thread
 * enqueued (for accounting in benchmarks). */
int32_t nslm_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* NSLM_H */
