/*
 * dart.h -- C ABI of libdart.so, the sm_100a implementation of the DART layer
 * hot path ("DART: Decoded Attention over Recurrent States for Efficient
 * Long-Context Sequence Modeling").
 *
 * Three compute entry points, one per stage of the layer:
 *   dart_ssd_chunk_scan  Mamba-2 SSD chunked scan that also writes out every
 *                        chunk's state contribution dH[c] (the chunk memory);
 *   dart_sma_forward     state-memory attention over those memories plus the
 *                        gated residual;
 *   dart_decode_step     one new token per sequence against the cache of
 *                        chunk memories and the recurrent state.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Notation: B batch, L sequence length, H heads, P head dimension (value
 *   axis), N state size (key axis), S chunk size, C = ceil(L / S) chunks (a
 *   partial last chunk counts), G = ngroups groups of heads sharing one B
 *   and one C projection (Mamba-2's grouped B/C): G divides H and head h
 *   reads group h / (H / G).  G = 1 is one B and C for all heads.
 * - Every tensor is dense, row-major (last index fastest), on the CUDA device
 *   that is current for the calling thread, and 16-byte aligned.  Layouts:
 *     x[B,L,H,P]  dt[B,L,H]  A[H]  Bm[B,L,G,N]  Cm[B,L,G,N]  Q[B,L,H,N]
 *     E[B,L,H,P]  y[B,L,H,P]  dH[B,H,C,N,P]  states[B,H,C,N,P]
 * - dtype selects the element type of x, Bm, Cm, Q, E and of the chunk
 *   memories dH / the decode cache: DART_F32 (float) or DART_BF16
 *   (__nv_bfloat16).  dt, A, y, states, the decode state and dH_cur are
 *   always float.  Accumulation is always float.
 * - Ownership: the caller allocates and owns every buffer, including the
 *   workspaces.  The library's own device memory is a status word per device
 *   and the fixed 16 MiB scratch array of dart_decode_step_noalloc; both are
 *   statically sized, exist on every device where the library's module is
 *   loaded, and live until the process exits.
 * - Execution: calls enqueue kernels on `stream` (a cudaStream_t; NULL is the
 *   legacy default stream) and return without synchronising.  Arguments are
 *   validated on the host before anything is enqueued; a rejected call
 *   enqueues nothing and returns DART_ERR_INVALID_ARG or
 *   DART_ERR_UNSUPPORTED, with a message in dart_last_error().  Conditions
 *   only the device can see (a decode counter out of range, a bounded wait
 *   that gave up) are latched in the device status word and reported by
 *   dart_sync_status().  Nothing traps.
 * - Thread safety: calls may be made from several host threads; each thread
 *   has its own dart_last_error() message.
 */
#ifndef DART_H_
#define DART_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DART_OK = 0,
    DART_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, bad counter */
    DART_ERR_UNSUPPORTED = 2,  /* valid but not compiled: (N, P, S, dtype) combination */
    DART_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    DART_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up */
    DART_ERR_DEVICE = 5        /* the device flagged bad state (e.g. decode cache full) */
} dart_status;

typedef enum { DART_F32 = 0, DART_BF16 = 1 } dart_dtype;

typedef struct {
    int batch;    /* B (decode: number of sequences) */
    int seqlen;   /* L >= 1 (ignored by dart_decode_step); C = ceil(L / chunk) chunks */
    int nheads;   /* H */
    int headdim;  /* P, the value axis */
    int dstate;   /* N, the key axis */
    int chunk;    /* S */
    int ngroups;  /* G >= 1, dividing nheads: B and C groups of heads; an
                     invalid count returns DART_ERR_INVALID_ARG */
} dart_dims;

/*
 * Workspace for dart_ssd_chunk_scan, in bytes: B*H*C floats (the per-chunk
 * sum of log-decays, padded to 256 bytes); for the bf16 shapes that run on
 * the tensor cores also the bf16 state entering each chunk (B*H*C*N*P*2
 * bytes) and three fp32 per-token decay terms (3*B*H*C*S*4 bytes).  Pass at
 * least this many bytes, 16-byte aligned.
 * Its contents on entry do not matter and are not preserved.
 */
size_t dart_ssd_chunk_scan_workspace_bytes(const dart_dims* dims, dart_dtype dtype);

/*
 * Mamba-2 SSD chunked scan with retained chunk memories.
 *
 * Computes, per batch b and head h (Mamba-2 "Transformers are SSMs" SSD view,
 * Eq. (4), which the DART pages build on; Pith review of DART, "What carries
 * the argument"):
 *   recurrence   H_t = exp(dt_t A_h) H_{t-1} + dt_t B_t x_t^T,  H_{-1} = init
 *   output       y_ssd_t = H_t^T C_t   (the state already includes token t)
 *   memory       dH[c] = sum_{s in chunk c} exp(sum_{r=s+1}^{e(c)} dt_r A_h)
 *                         dt_s B_s x_s^T    (what chunk c adds to the state at
 *                         its last token e(c); no decay beyond e(c))
 *   boundary     states[c] = H_{e(c)}
 * evaluated chunk-wise (intra-chunk quadratic block + inter-chunk state
 * passing), not token by token.  C = ceil(L / S): when L is not a multiple
 * of S the last chunk is partial and closes at e(C-1) = L-1, so its dH and
 * state are what a decode carries on from (dH_cur = dH[C-1], state =
 * states[C-1], C-1 cached memories, position L mod S).
 *
 *   x, Bm, Cm     dtype inputs; dt, A float inputs (dt > 0 after softplus,
 *                 A < 0 per head).
 *   init_state    nullable float [B,H,N,P]; NULL means zero.
 *   y_ssd         float [B,L,H,P] output.
 *   dH            dtype [B,H,C,N,P] output (rounded to nearest-even for bf16).
 *   states        float [B,H,C,N,P] output.
 *   workspace     device scratch of dart_ssd_chunk_scan_workspace_bytes().
 * Requires (N, P, S, dtype) in the compiled set (see
 * dart_supported()).
 */
dart_status dart_ssd_chunk_scan(const dart_dims* dims, dart_dtype dtype,
                                const void* x, const float* dt, const float* A,
                                const void* Bm, const void* Cm, const float* init_state,
                                float* y_ssd, void* dH, float* states,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * State-memory attention with the gated residual (Pith review of DART, "Core
 * claim" and "What carries the argument"; SMA Eqs. (5)-(10)).  For token t in
 * chunk k(t) = t / S and each chunk c < k(t):
 *   value  v_{t,c} = C_t^T dH[c]            (P)
 *   key    k_{t,c} = dH[c] E_t              (N)
 *   score  s_{t,c} = Q_t . k_{t,c} / sqrt(N)
 *   o_t = sum_c softmax_c(s_{t,c}) v_{t,c};   o_t = 0 when k(t) == 0.
 * Memories are used as stored, without inter-chunk decay (referee comment 3
 * on Eq. (8)).  With a partial last chunk (L not a multiple of S) dH has
 * C = ceil(L / S) memories and no token attends to the last one.
 *   out = y_ssd + g * o   when y_ssd != NULL (the DART layer output), else
 *   out = o               (the raw readout).
 *   Q[B,L,H,N], E[B,L,H,P], Cm[B,L,G,N], dH[B,H,C,N,P]: dtype inputs.
 *   y_ssd: nullable float [B,L,H,P]; out: float [B,L,H,P], either the same
 *   pointer as y_ssd (updated in place, the fastest form) or not overlapping it
 *   (y_ssd is then copied into out on the stream first).
 */
dart_status dart_sma_forward(const dart_dims* dims, dart_dtype dtype,
                             const void* Q, const void* E, const void* Cm, const void* dH,
                             float g, const float* y_ssd, float* out, void* stream);

/*
 * Workspace for dart_sma_forward_decayed, in bytes: the per-token in-chunk
 * log-decay prefix (B*H*C*S floats, padded to 256 bytes) and the per-chunk
 * prefix of chunk log-decays (B*H*C doubles).  0 for invalid dims.
 */
size_t dart_sma_decayed_workspace_bytes(const dart_dims* dims);

/*
 * Decayed-memory variant of dart_sma_forward (referee major comment 3 on SMA
 * Eq. (8), Pith review of DART: the memories carried to the query token by
 * the recurrence's decay instead of used raw).  For token t in chunk k(t)
 * and each c < k(t) memory c is first scaled by
 *   w_{t,c} = exp( A_h * sum_{r=e(c)+1}^{t} dt_r ),   e(c) = (c+1) S - 1,
 * the share of dH[c] still present in the SSM state at t, and then used as
 * in dart_sma_forward for both the key and the value:
 *   s_{t,c} = w_{t,c} Q_t . (dH[c] E_t) / sqrt(N),  v_{t,c} = w_{t,c} C_t^T dH[c].
 *   dt [B,L,H], A [H]: float, the same tensors the scan was given.
 *   workspace: device scratch of dart_sma_decayed_workspace_bytes(), 16-byte
 *   aligned; contents on entry do not matter and are not preserved.
 * Other arguments, layouts, output modes and errors as dart_sma_forward.
 * Enqueues the two decay-prefix kernels before the attention kernel.
 */
dart_status dart_sma_forward_decayed(const dart_dims* dims, dart_dtype dtype,
                                     const void* Q, const void* E, const void* Cm, const void* dH,
                                     const float* dt, const float* A, float g, const float* y_ssd,
                                     float* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace for dart_ssd_scan_backward, in bytes: the recomputed states of
 * one chunk per (b, h) (2 * B*H*S*N*P floats), per-head dB and dC
 * (2 * B*L*H*N floats) and per-(b, h) dA, each padded to 256 bytes.
 */
size_t dart_ssd_scan_backward_workspace_bytes(const dart_dims* dims);

/*
 * Gradients through dart_ssd_chunk_scan (the training pass, DART abstract
 * "DART supports practical training"; the recurrence of Eq. (4) of the SSD
 * view).  For loss = sum(dy * y_ssd) + sum(ddH * dH), with a_t = exp(dt_t A_h)
 * and the adjoints run from the last token,
 *   G_t = C_t dy_t^T + a_{t+1} G_{t+1}                     (dLoss/dH_t)
 *   K_t = ddH[c] at the chunk's last token, a_{t+1} K_{t+1} inside the chunk
 *   dx_t = dt_t (G_t + K_t)^T B_t,  dB_t = sum_h dt_t (G_t + K_t) x_t,
 *   dC_t = sum_h H_t dy_t,
 *   ddt_t = sum((G_t + K_t) o B_t x_t^T) + A_h a_t (sum(G_t o H_{t-1}) + sum(K_t o D_{t-1})),
 *   dA_h = sum over b, t of dt_t a_t (sum(G_t o H_{t-1}) + sum(K_t o D_{t-1})),
 *   dinit_state = a_0 G_0,
 * D the chunk-restarted accumulator whose value at a chunk's last token is
 * dH[c].  The forward's H_{t-1} are recomputed chunk by chunk from `states`.
 *   x, Bm, Cm: dtype, dt, A, init_state (nullable): float -- the forward's inputs;
 *   states: float [B,H,C,N,P] the forward's boundary states;
 *   dy: float [B,L,H,P]; ddH: nullable float [B,H,C,N,P] (NULL = zero), e.g.
 *   dart_sma_backward's memory gradient;
 *   dCm_add: nullable float [B,L,G,N], added to dCm (NULL = nothing); passing
 *   dart_sma_backward's dCm gives the layer's C gradient.  It may be dCm
 *   itself (each element is read before it is written);
 *   dx float [B,L,H,P], ddt float [B,L,H], dA float [H], dBm, dCm float [B,L,G,N] (summed over the heads of each group);
 *   dinit_state: nullable float [B,H,N,P].
 * CUDA cores, one CTA per (b, h); sums in a fixed order (deterministic).
 * Compiled for (N, P) = (128, 64), (64, 64), (16, 16).
 */
dart_status dart_ssd_scan_backward(const dart_dims* dims, dart_dtype dtype,
                                   const void* x, const float* dt, const float* A,
                                   const void* Bm, const void* Cm, const float* init_state,
                                   const float* states, const float* dy, const float* ddH,
                                   const float* dCm_add,
                                   float* dx, float* ddt, float* dA, float* dBm, float* dCm,
                                   float* dinit_state, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Workspace for dart_sma_backward, in bytes: the softmax weights and score
 * gradients of every (token, memory) pair (2 * B*H*L*C floats), the per-head
 * dC (B*L*H*N floats) and per-tile dg partials, each padded to 256 bytes.
 * 0 for invalid dims.
 */
size_t dart_sma_backward_workspace_bytes(const dart_dims* dims);

/*
 * Gradients of state-memory attention with the gated residual (the training
 * pass, DART abstract "DART supports practical training"; the forward of
 * dart_sma_forward with raw memories).  Given dy = dLoss/dy for
 * y = y_ssd + g o, with do = g dy_t, p the softmax over the memories c < k(t),
 * v_c = C_t^T dH[c], w1 = dH[c] E_t, w2 = dH[c] do and D_t = do . o_t:
 *   ds_c = p_c (C_t . w2 - D_t)
 *   dQ_t = sum_c ds_c w1 / sqrt(N)         dE_t = sum_c ds_c dH[c]^T Q_t / sqrt(N)
 *   dC_t = sum_h sum_c p_c w2              dg = sum dy . o
 *   ddH[c] = sum_{t: k(t) > c} (ds_tc / sqrt(N) Q_t E_t^T + p_tc C_t do_t^T)
 * (dy also flows unchanged to y_ssd; that part is the caller's.)
 *   Q[B,L,H,N], E[B,L,H,P], Cm[B,L,G,N], dH[B,H,C,N,P]: dtype inputs (as given
 *   to the forward); dy: float [B,L,H,P].
 *   dQ float [B,L,H,N], dE float [B,L,H,P], dCm float [B,L,G,N],
 *   ddH float [B,H,C,N,P], dg float [1]: outputs, every element written.
 *   workspace: device scratch of dart_sma_backward_workspace_bytes().
 * CUDA-core kernels; sums run in a fixed order (deterministic).  Shapes and
 * errors as dart_sma_forward.
 */
dart_status dart_sma_backward(const dart_dims* dims, dart_dtype dtype,
                              const void* Q, const void* E, const void* Cm, const void* dH,
                              float g, const float* dy, float* dQ, float* dE, float* dCm,
                              float* ddH, float* dg, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Workspace for dart_decode_step: per (sequence, head, split) partial softmax
 * statistics and partial outputs.  Pass at least this many bytes.  Every
 * decode entry takes 1 <= cmax <= 2^20 (memories per sequence) and rejects
 * other values with DART_ERR_INVALID_ARG; this query returns 0 for them.
 */
size_t dart_decode_step_workspace_bytes(const dart_dims* dims, dart_dtype dtype, int cmax);

/*
 * One decode step for dims->batch sequences (DART abstract and Pith review
 * "If this is right": the length-dependent inference cache is the set of
 * chunk memories).  Per sequence b and head h, with n = n_chunks[b] completed
 * memories and pos = pos[b] the index of the incoming token inside its chunk:
 *   a = exp(dt A_h);  state = a state + dt B x^T;  dH_cur = a dH_cur + dt B x^T
 *   y = state^T C + g * SMA(Q, E, C; dH_cache[b,h,0..n-1])
 *   if pos == S-1:  dH_cache[b,h,n] = dH_cur (rounded to dtype);
 *                   dH_cur = 0;  n_chunks[b] = n + 1;  pos[b] = 0
 *   else            pos[b] = pos + 1
 *   x_t[B,H,P], B_t[B,G,N], C_t[B,G,N], Q_t[B,H,N], E_t[B,H,P]: dtype inputs;
 *   dt_t[B,H], A[H]: float inputs.
 *   state, dH_cur: float [B,H,N,P], in/out.
 *   dH_cache: dtype [B,H,cmax,N,P], in/out (slots >= n are not read).
 *   n_chunks, pos: int32 [B] device arrays, in/out.
 *   y: float [B,H,P] output.
 * A sequence whose counters are out of range (n > cmax, pos outside [0,S),
 * or an append with n == cmax) produces no output update for that sequence,
 * leaves its state untouched and latches DART_ERR_DEVICE.
 */
dart_status dart_decode_step(const dart_dims* dims, dart_dtype dtype,
                             const void* x_t, const float* dt_t, const float* A,
                             const void* B_t, const void* C_t, const void* Q_t, const void* E_t,
                             float g, float* state, float* dH_cur, void* dH_cache, int cmax,
                             int* n_chunks, int* pos, float* y,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * dart_decode_step with decayed memories (referee major comment 3 on SMA
 * Eq. (8), Pith review of DART; the decode form of dart_sma_forward_decayed).
 * mem_logdecay: float [B,H,cmax], in/out.  Slot c < n_chunks[b] holds the
 * log-decay memory c has accumulated since its chunk closed,
 *   lw_c = sum_{r=e(c)+1}^{t-1} dt_r A_h   (t the incoming token).
 * The step sets lw_c += dt_t A_h, scales the memory's score and value by
 * exp(lw_c) exactly as dart_sma_forward_decayed does, and when the token
 * closes its chunk sets the appended memory's slot to 0.  Slots >= n_chunks
 * are not read.  Everything else -- arguments, layouts, counters, errors --
 * as dart_decode_step.
 */
dart_status dart_decode_step_decayed(const dart_dims* dims, dart_dtype dtype,
                                     const void* x_t, const float* dt_t, const float* A,
                                     const void* B_t, const void* C_t, const void* Q_t,
                                     const void* E_t, float g, float* state, float* dH_cur,
                                     void* dH_cache, int cmax, int* n_chunks, int* pos,
                                     float* mem_logdecay, float* y,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * mem_logdecay for decode after a prefill of dims->seqlen = L tokens (the
 * handoff of dart_ssd_chunk_scan: L / S completed memories are cached):
 *   mem_logdecay[b,h,c] = sum_{r=(c+1)S}^{L-1} dt[b,r,h] A[h]   for c < L / S,
 * summed with an fp64 carry; other slots are left as they are.
 *   dt: float [B,L,H] (the prefill's), A: float [H], mem_logdecay: float
 *   [B,H,cmax] with L / S <= cmax.  Uses batch, seqlen, nheads and chunk of
 *   dims.  One kernel on `stream`.
 */
dart_status dart_decode_memlog_init(const dart_dims* dims, const float* dt, const float* A,
                                    float* mem_logdecay, int cmax, void* stream);

/*
 * dart_decode_step with an fp8 cache: each row of P values of a cached
 * memory is stored as OCP FP8 E4M3 codes times 2^k, one signed exponent k
 * per row -- half the bytes of a bf16 cache, and the decode step streams the
 * cache, so about half the time (the cache quantization the pages list as
 * an extension; the cache itself is the DART abstract's and the Pith
 * review's "If this is right").
 *   cache:     uint8 [B,H,cmax,N,P] E4M3 codes, in/out;
 *   cache_exp: int8  [B,H,cmax,N] row exponents, in/out; memory row value =
 *              code_value * 2^k.
 * The step reads memories 0..n-1 dequantized.  When the token closes its
 * chunk the finished contribution is quantized row by row into slot n:
 * k = the smallest integer with max|row| * 2^-k <= 448, clamped to
 * [-126, 60], codes = E4M3(row * 2^-k) rounded to nearest even and
 * saturating at 448.  mem_logdecay: NULL for raw memories, else as in
 * dart_decode_step_decayed.  Inputs x_t .. E_t in dtype (bf16 or f32); the
 * remaining arguments, counters and errors as dart_decode_step.  Compiled
 * for P = 64 with N = 64 or 128.  Contributions to the value readout below
 * 2^-89 in magnitude underflow to zero.
 */
dart_status dart_decode_step_e4m3(const dart_dims* dims, dart_dtype dtype,
                                  const void* x_t, const float* dt_t, const float* A,
                                  const void* B_t, const void* C_t, const void* Q_t, const void* E_t,
                                  float g, float* state, float* dH_cur, unsigned char* cache,
                                  signed char* cache_exp, int cmax, int* n_chunks, int* pos,
                                  float* mem_logdecay, float* y,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The prefill -> fp8 decode handoff: memories 0..nmem-1 of dH (dtype
 * [B,H,C,N,P] as written by dart_ssd_chunk_scan, C = ceil(seqlen / chunk))
 * quantized into cache slots 0..nmem-1 of an E4M3 cache (layouts and
 * rounding as dart_decode_step_e4m3).  Uses batch, seqlen, nheads, headdim,
 * dstate and chunk of dims; nmem <= min(C, cmax).  One kernel on `stream`.
 */
dart_status dart_cache_quantize_e4m3(const dart_dims* dims, dart_dtype dtype, const void* dH, int nmem,
                                     unsigned char* cache, signed char* cache_exp, int cmax, void* stream);

/*
 * dart_decode_step for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is an interface for embedding the decode
 * step where cudaMalloc is not available to the caller -- for example a host
 * runtime that owns all device memory and hands out only preallocated
 * tensors, or a serving loop that must not call into the allocator (which
 * may synchronise the device) between steps.
 *
 * Same arguments, computation and device-side error behaviour as
 * dart_decode_step, without the workspace: the per-(sequence, head, split)
 * partial results live in a 16 MiB array that the library keeps in static
 * device memory, one per device that loads the library, held until the
 * process exits.  The caller still passes every input and output.
 *   - Limit: dart_decode_step_workspace_bytes(dims, dtype, cmax) must be at
 *     most 16 MiB (16777216 bytes); larger batches are rejected with
 *     DART_ERR_UNSUPPORTED and a message giving both sizes.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - Every call shares the one array: calls that overlap on the GPU (on
 *     different streams, or from several threads without ordering) race.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
dart_status dart_decode_step_noalloc(const dart_dims* dims, dart_dtype dtype,
                                     const void* x_t, const float* dt_t, const float* A,
                                     const void* B_t, const void* C_t, const void* Q_t,
                                     const void* E_t, float g, float* state, float* dH_cur,
                                     void* dH_cache, int cmax, int* n_chunks, int* pos, float* y,
                                     void* stream);

/*
 * 1 when (dstate N, headdim P, chunk S, dtype) is compiled in, else 0.
 */
int dart_supported(int dstate, int headdim, int chunk, dart_dtype dtype);

/*
 * Name of the kernel dart_sma_forward dispatches to for this shape and dtype
 * ("sma_simt" on CUDA cores, "sma_tcgen05" on the tensor cores), or "" when
 * the combination is not compiled.  The string is static.
 */
const char* dart_sma_impl(int dstate, int headdim, int chunk, dart_dtype dtype);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: DART_OK, DART_ERR_TIMEOUT or DART_ERR_DEVICE (or
 * DART_ERR_CUDA if the synchronisation itself failed).
 */
dart_status dart_sync_status(void* stream);

/*
 * Failure-detection drill: launches one warp that waits, through the bounded
 * mbarrier wait every tensor-core kernel uses, on an mbarrier nothing
 * arrives on.  After limit_us microseconds (1 .. 2e6) the wait gives up and
 * latches the timeout in the status word (kernel 9, wait site 1); nothing
 * else is in flight, so the next dart_sync_status(stream) returns
 * DART_ERR_TIMEOUT, clears the word, and later calls run clean.  Returns
 * DART_OK once launched, DART_ERR_INVALID_ARG for a limit out of range.
 */
dart_status dart_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Message describing the last failure on the calling host thread ("" if none). */
const char* dart_last_error(void);

/* ABI version, bumped on any signature change or addition (2: the decayed-memory,
 * E4M3-cache and backward entry points; 3: dCm_add of the scan backward and
 * ngroups; 4: dart_selftest_wait_timeout). */
int dart_abi_version(void);

/*
 * Number of CUDA kernels this library has enqueued since it was loaded
 * (process-wide, all devices and threads).  Lets a caller count the launches
 * inside a region without a profiler.
 */
unsigned long long dart_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DART_H_ */
