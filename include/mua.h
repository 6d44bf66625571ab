/*
 * mua.h — C ABI of libmua.so, a B200 (sm_100a) implementation of the MicroAdam
 * optimizer step.
 *
 * [MicroAdam ¶n] is paragraph n of the web page "MicroAdam (Sparse-Gradient
 * Adaptive Optimization with Quantized Error Feedback)". ¶1 defines the step:
 *   a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t)              (dequantize + add)
 *   (I_t, V_t) = T_k(|a_t|) per block of B_d < 2^15 - 1    (block Top-k, int16 I)
 *   a_t[I_t] = 0; e_{t+1} = Q(a_t, delta_{t+1}, Delta_{t+1}) (4-bit error feedback)
 *   G[t mod m] = (I_t, V_t)                                  (circular window)
 *   m_hat = AdamStats(beta1, G), v_hat = AdamStats(beta2, G^2),
 *   AdamStats: z[I_i] += beta^r V_i over the window rows (r = row age),
 * followed by the update p <- p - lr * m_hat / (eps + sqrt(v_hat)) on the
 * window's index union. ¶2 gives the state size 0.5d + 4mk bytes.
 *
 * Conventions for every entry point:
 *  - Device memory is owned by the caller. The library never allocates,
 *    frees or synchronizes device memory inside a step; a handle (mua_t)
 *    holds host-side geometry only.
 *  - "device pointer" arguments must point to memory of the current CUDA
 *    device; "host pointer" arguments to host memory.
 *  - Work is enqueued on the given cudaStream_t (passed as void*; NULL is the
 *    legacy default stream). Calls return once the work is enqueued.
 *  - Return value: MUA_OK (0) or a negative MUA_ERR_* code; mua_strerror()
 *    names it and, for MUA_ERR_CUDA, mua_last_cuda_error() gives the CUDA
 *    runtime's message. No exception or abort crosses the ABI.
 *  - Device-side anomalies (a non-finite a_t) never trap: they set bits of a
 *    sticky status word inside the state, read by mua_get_status().
 *  - One handle may be used by several threads only if calls on the same
 *    state buffer are serialized (the state is updated in place).
 */
#ifndef MUA_H
#define MUA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUA_OK 0
#define MUA_ERR_ARG (-1)         /* an argument is out of range or NULL            */
#define MUA_ERR_UNSUPPORTED (-2) /* a valid request this build does not implement  */
#define MUA_ERR_ALIGN (-3)       /* a device pointer is not 16-byte aligned         */
#define MUA_ERR_CUDA (-4)        /* the CUDA runtime reported an error              */

/* Status bits (sticky, in the state header). */
#define MUA_STATUS_NONFINITE 1u  /* some a_t was NaN or +-inf; results unspecified  */
#define MUA_STATUS_TIMEOUT 2u    /* a CTA of the fused step gave up waiting at its grid
                                    barrier (see mua_set_wait_limit_ns); that step's
                                    results are unspecified                           */

/* Fields written by mua_state_layout(). */
#define MUA_LAYOUT_HEADER 0      /* byte offset of the 256-byte scalar header        */
#define MUA_LAYOUT_CODES 1       /* byte offset of the packed 4-bit codes e          */
#define MUA_LAYOUT_WINDOW 2      /* byte offset of the window G                      */
#define MUA_LAYOUT_ROW_STRIDE 3  /* uint32 entries per (block, row): k_b rounded to 4 */
#define MUA_LAYOUT_BLOCKS 4      /* number of blocks n_b                             */
#define MUA_LAYOUT_BYTES 5       /* total state bytes (= mua_state_bytes)            */
#define MUA_LAYOUT_FIELDS 6

typedef struct mua_ctx* mua_t;

/*
 * mua_create — describe one flat parameter vector of d fp32 values, cut into
 * n_b = ceil(d / B_d) blocks [MicroAdam ¶1]. Host only; touches no GPU.
 *   d            number of parameters, >= 1
 *   block_size   B_d, even, 2 <= B_d <= 32766 (int16 block-relative indices,
 *                B_d < 2^15 - 1 [MicroAdam ¶1])
 *   k_per_block  k_b, 1 <= k_b <= B_d; a ragged last block of length L keeps
 *                ceil(L * k_b / B_d) entries
 *   window       m, 1 <= m <= 64 rows in the circular window G
 *   bits         b, must be 4 (MUA_ERR_UNSUPPORTED otherwise)
 *   out          receives the handle (release with mua_destroy)
 * Errors: MUA_ERR_ARG for out-of-range values or NULL out;
 * MUA_ERR_UNSUPPORTED when bits != 4 or when the window of one block,
 * m * k_b entries, is too large for the on-chip AdamStats (m * k_b rounded up
 * to a multiple of 4 per row, more than 15360 entries).
 */
int mua_create(int64_t d, int32_t block_size, int32_t k_per_block, int32_t window,
               int32_t bits, mua_t* out);

/*
 * mua_create_shard — like mua_create, for the contiguous run of blocks
 * [block_begin, block_begin + block_count) of a d_total-parameter vector, as
 * one rank of a sharded step holds it. Random draws use global element
 * indices, so the shards of a vector reproduce the unsharded step exactly
 * once the ranks combine their (delta, Delta) partials between mua_select and
 * mua_apply (see mua_minmax_offset). Host only.
 */
int mua_create_shard(int64_t d_total, int32_t block_size, int32_t k_per_block,
                     int32_t window, int32_t bits, int64_t block_begin,
                     int64_t block_count, mua_t* out);

/*
 * mua_create_segmented — like mua_create for a tensor list: the d-vector is
 * the concatenation of n_seg tensors of lengths seg_len[0..n_seg) (d is their
 * sum, elements in list order), and each tensor is cut into its own blocks of
 * B_d, the last one ragged (k = ceil(L * k_b / B_d) entries), so no block spans
 * two tensors. delta and Delta stay global over the d-vector [MicroAdam ¶1].
 * Blocks are numbered tensor by tensor; the state layout, window rows and
 * random draws (by global element index) are those of the flat case with that
 * block count. seg_len is read during the call only. Host only.
 * Errors: MUA_ERR_ARG for NULL pointers, n_seg < 1, a length < 1 or the
 * arguments mua_create rejects; MUA_ERR_UNSUPPORTED for an odd length (a
 * block must start on a byte of the 4-bit codes), n_seg > MUA_MAX_SEGMENTS,
 * and what mua_create cannot hold. The 16-byte vector path is used when B_d
 * and every length are multiples of 8.
 */
#define MUA_MAX_SEGMENTS 512
int mua_create_segmented(const int64_t* seg_len, int32_t n_seg, int32_t block_size,
                         int32_t k_per_block, int32_t window, int32_t bits, mua_t* out);

/* mua_destroy — release a handle (NULL is ignored). Host only. */
void mua_destroy(mua_t h);

/*
 * mua_state_bytes — size of the optimizer state buffer for this handle:
 * 256 (header) + ceil(d/2) rounded up to 256 (4-bit codes, 0.5d [MicroAdam
 * ¶2]) + 4 * n_b * m * round_up(k_b, 4) (window, 4mk [MicroAdam ¶2]).
 * The caller allocates this many bytes of device memory, 16-byte aligned,
 * and zero-fills it before the first step (zero state = e_0 = 0,
 * delta = Delta = 0, empty window). Returns a negative code on a NULL handle.
 */
int64_t mua_state_bytes(mua_t h);

/*
 * mua_state_layout — write the MUA_LAYOUT_FIELDS int64 values above into the
 * host array out. The window is uint32[n_b][m][row_stride]: entry = int16 I
 * (low half; 0xFFFF = empty slot) | bf16 V << 16; row (t mod m) of block j
 * holds the block's Top-k of step t: its k entries first, in an order the
 * kernels fix from the data alone (the same bytes on every run; the method
 * does not order a row, and no later use of it depends on the order), then
 * empty slots. The header
 * holds two (-delta, Delta) fp32 pairs at words 0-1 and 2-3 (pair t mod 2 is
 * step t's (delta_t, Delta_t)), the status word at word 4 and the fused step's
 * barrier count at word 5 (reset by every fused step).
 */
int mua_state_layout(mua_t h, int64_t* out);

/*
 * mua_step — one full MicroAdam step t [MicroAdam ¶1] on `stream`.
 * For a whole vector (not a shard) of blocks of at most 16384 entries whose
 * CTAs the current device can all hold at once (up to one block per SM), the
 * step is ONE cooperative launch that keeps a_t in registers across a
 * grid-wide barrier (bounded: see mua_set_wait_limit_ns); otherwise it is
 * mua_select followed by mua_apply. Both give the same bytes.
 * mua_step_launches tells which applies.
 *   params  device, fp32[d], updated in place
 *   grads   device, bf16[d] (raw 16-bit patterns), read only
 *   state   device, mua_state_bytes(h) bytes, updated in place
 *   lr, beta1, beta2, eps, wd   fp32 hyper-parameters, all finite;
 *           0 <= beta < 1; eps > 0 (an index whose window values are all
 *           zero would otherwise divide 0 by 0); wd is decoupled weight decay
 *           applied to every parameter as p *= (1 - lr*wd) before the update
 *   t       step number: 1 for the first step, then t+1 on every call
 *   seed    key of the Philox4x32-10 stream of the stochastic rounding
 * Errors: MUA_ERR_ARG (NULL pointer, t < 1, bad hyper-parameter),
 * MUA_ERR_ALIGN (a pointer not 16-byte aligned), MUA_ERR_CUDA.
 */
int mua_step(mua_t h, float* params, const uint16_t* grads, void* state, float lr,
             float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
             void* stream);

/*
 * mua_step_bf16 — mua_step for bf16 parameters: params is bf16[d] (raw
 * 16-bit patterns, device, 16-byte aligned), updated in place; there is no
 * fp32 copy. Every parameter the step changes (the window's index union, and
 * with wd != 0 every parameter) is computed in fp32 from its bf16 value and
 * rounded once to bf16, to nearest with ties to even: the page's full
 * fine-tune of LLaMA-2 7B on a single 40 GB GPU [MicroAdam ¶4] leaves no room
 * for 27 GB of fp32 parameters. Everything else (state, window, codes) is that
 * of mua_step. Arguments and errors as mua_step.
 */
int mua_step_bf16(mua_t h, uint16_t* params, const uint16_t* grads, void* state, float lr,
                  float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
                  void* stream);

/*
 * mua_select — first half of step t [MicroAdam ¶1]: stages (1)-(3) and (5):
 * a_t from grads and e_t, the per-block Top-k written to row t mod m of G,
 * and the per-block residual min/max folded into the (-delta_{t+1},
 * Delta_{t+1}) pair of the header (reset first, see mua_minmax_offset).
 * params, mhat and vhat are not touched: params may be NULL (for bf16
 * parameters pass NULL); non-NULL pointers are checked for alignment.
 * mua_select(t) and mua_apply(t) must be called in that order with identical
 * arguments; a sharded caller all-reduces the header pair between them.
 * Arguments and errors as mua_step.
 */
int mua_select(mua_t h, float* params, const uint16_t* grads, void* state, float lr,
               float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
               float* mhat, float* vhat, void* stream);

/*
 * mua_minmax_offset — byte offset in the state of the two fp32 words
 * (-delta_{t+1}, Delta_{t+1}) that mua_select(t) produces. Both are >= +0, so
 * a sharded caller combines the ranks' partials with an all-reduce MAX over
 * the two words read as uint32. Host only; negative code on bad arguments.
 */
int64_t mua_minmax_offset(mua_t h, int64_t t);

/*
 * mua_apply — second half of step t after mua_select(t): stage (4), the
 * quantization of the residual into e_{t+1} with (delta_{t+1}, Delta_{t+1}),
 * and stage (6), the AdamStats update of the parameters. If mhat / vhat are
 * non-NULL (device, fp32[d]), m_hat and v_hat are also written at every index
 * of the window's union (other entries are left untouched), for testing and
 * diagnostics. Arguments and errors as mua_step.
 */
int mua_apply(mua_t h, float* params, const uint16_t* grads, void* state, float lr,
              float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
              float* mhat, float* vhat, void* stream);

/*
 * mua_apply_bf16 — mua_apply for bf16 parameters (see mua_step_bf16).
 */
int mua_apply_bf16(mua_t h, uint16_t* params, const uint16_t* grads, void* state, float lr,
                   float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
                   float* mhat, float* vhat, void* stream);

/*
 * mua_step_launches — kernel launches mua_step(h, ...) (bf16_params == 0) or
 * mua_step_bf16(h, ...) (bf16_params != 0) makes on the current device: 1
 * (the fused one-launch step) or 2 (mua_select + mua_apply). Queries the
 * device once per device, handle and parameter type. Returns MUA_ERR_ARG for
 * a NULL handle, MUA_ERR_CUDA if the query fails.
 */
int mua_step_launches(mua_t h, int32_t bf16_params);

/*
 * mua_set_wait_limit_ns — bound, in nanoseconds of the GPU's global timer, on
 * how long a CTA of the fused step waits at its grid barrier before it sets
 * MUA_STATUS_TIMEOUT and returns without finishing the step (default 2 s,
 * far above a step's duration; the CTAs of a cooperative launch are all
 * resident, so the wait normally ends in microseconds). A limit <= 0 makes a
 * CTA give up as soon as it would wait: a way to exercise that path in tests.
 * Host only; MUA_ERR_ARG for a NULL handle.
 */
int mua_set_wait_limit_ns(mua_t h, int64_t ns);

/*
 * mua_get_status — copy the state's sticky status word (MUA_STATUS_* bits)
 * into the host integer *out, after the work already enqueued on `stream`.
 * Synchronizes `stream`. Returns MUA_ERR_ARG for NULL arguments and
 * MUA_ERR_CUDA if the copy fails.
 */
int mua_get_status(mua_t h, const void* state, void* stream, int32_t* out);

/* mua_strerror — static text for a return code. */
const char* mua_strerror(int code);

/* mua_last_cuda_error — text of the last CUDA error seen by this thread. */
const char* mua_last_cuda_error(void);

/* mua_version — library version string. */
const char* mua_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUA_H */
