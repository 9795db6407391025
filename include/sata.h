/*
 * sata.h — C ABI of the B200 (sm_100a) library for causal SATA attention
 * (symmetry-aware Taylor approximation).
 *
 * Operation.  Per head, with s_ij = q_i . k_j / sqrt(dK) and
 * T_P(s) = sum_{p=0}^{P-1} s^p / p!  (exp truncated to degrees 0..P-1):
 *     out_i = sum_{j<=i} T_P(s_ij) v_j  /  sum_{j<=i} T_P(s_ij)
 * evaluated through the feature map over the minimal basis of each order-p
 * symmetric tensor (index tuples i_1 <= ... <= i_p, the tables M_p) and a
 * fixed-size state S of shape [m, dV+1], m = C(dK+P-1, P-1), whose last column
 * is the normaliser.
 *   Source: "对称性感知泰勒近似注意力机制的恒定计算成本工程实现" (blog.hotdry.top),
 *   sections "对称张量分解的核心洞察" (Taylor expansion, minimal basis
 *   C(dK+p-1,p), fixed index tables M_p) and "恒定计算成本的工程实现"
 *   (state of (dV+1) x C(dK+P-1,P-1) elements, per-token update and readout).
 *   Layout (batch, heads, seq, dim) and the dim**-0.5 scale follow
 *   "Transformer 注意力机制变体与长序列建模优化" (mokono.cn), section 2.1.
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device (or managed) memory of the current
 *     device, owned by the caller; the library never frees or retains them.
 *     Every base pointer must be 16-byte aligned.
 *   - Row-major contiguous layouts:
 *       q, k   [B, H, N, dK]     dtype = SATA_F32 (float) or SATA_BF16 (bfloat16)
 *       v      [B, H, N, dV]     same dtype as q, k
 *       out    [B, H, N, dV]     float
 *       state  [B, H, m, dV+1]   float; row r is basis row r in degree-major,
 *                                lexicographic order (the order of
 *                                sata_index_table); column dV is the normaliser
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous; no call synchronises the device except
 *     sata_get_error.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a status and launches nothing.  Nothing throws
 *     across this interface.
 *   - Supported: dK, dV in {8, 16, 32, 64}; 1 <= P <= 5 (P = 5 adds the
 *     degree-4 tensor: m = C(dK+4, 4), e.g. 814385 rows at dK = 64, and runs
 *     on CUDA cores); B, H, N >= 1 with B*H*N*max(dK,dV) < 2^31.
 *   - The library lazily allocates, per device, its basis tables and a
 *     grow-only scratch workspace (cudaMalloc); both live until sata_release()
 *     or process exit.  The first call on a device for a given (dK, P) builds
 *     the tables and waits for the device (cudaDeviceSynchronize): make it
 *     before any stream capture.
 *   - Thread safety: every prefill and decode call holds one internal
 *     (recursive) mutex from validation through its last launch, and the
 *     caches and the profiling records are read and written only under it,
 *     so calls from several host threads are serialised on the host (the
 *     work they enqueue runs in stream order on the GPU).
 *     sata_decode_step_noalloc is the exception; see its notes.
 */
#ifndef SATA_H_
#define SATA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sata_stream_t; /* == cudaStream_t */

typedef enum {
  SATA_OK = 0,
  SATA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, aliasing   */
  SATA_ERR_UNSUPPORTED = 2, /* dK, dV or P outside the supported set        */
  SATA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed          */
  SATA_ERR_NOMEM = 4,       /* workspace allocation failed                   */
  SATA_ERR_TIMEOUT = 5      /* a device-side bounded wait gave up            */
} sata_status;

typedef enum { SATA_F32 = 0, SATA_BF16 = 1 } sata_dtype;

/* Number of basis rows m = sum_{p<P} C(dK+p-1, p) = C(dK+P-1, P-1)
 * ("恒定计算成本的工程实现": state size (dV+1) x C(dK+P-1, P-1)).
 * Host only.  Returns -1 if dK < 1 or P < 1 or the result overflows int64. */
int64_t sata_basis_size(int dK, int P);

/* Writes M_p ("对称张量分解的核心洞察": index tuples of the upper-triangular
 * region), i.e. every tuple 0 <= i_1 <= ... <= i_p < dK in lexicographic
 * order, row-major [C(dK+p-1,p), p] int32, into host_out.  Host only.
 * cap_elems is the capacity of host_out in int32 elements.  Returns the number
 * of rows (>= 1; p = 0 has one empty row and writes nothing), or -1 on a bad
 * argument (dK < 1, p < 0, host_out NULL while p > 0) or when cap_elems is too
 * small (nothing is written then). */
int64_t sata_index_table(int dK, int p, int32_t *host_out, int64_t cap_elems);

/* Causal prefill from a zero state.  Writes out (every token) and overwrites
 * state with S after the last token.  q, k, v, out, state: see layouts above;
 * out and state must not overlap each other or the inputs.
 * Paths: bf16 inputs with P = 4 and dK = dV = 64 or dK = dV = 32 run on the
 * tcgen05 tensor cores (features and chunk-boundary states rounded to bf16,
 * in-chunk Taylor scores split into bf16 hi + lo parts, fp32 accumulation);
 * every other supported case runs in fp32 on CUDA cores.  With the environment variable
 * SATA_FORCE_SIMT=1 set before the first call, every prefill (and continued
 * prefill) takes the CUDA-core path, e.g. to cross-check the two paths.
 * Returns SATA_OK, SATA_ERR_INVALID_ARG, SATA_ERR_UNSUPPORTED, SATA_ERR_NOMEM
 * or SATA_ERR_CUDA. */
int sata_prefill(const void *q, const void *k, const void *v, float *out,
                 float *state, int B, int H, int N, int dK, int dV, int P,
                 sata_dtype dt, sata_stream_t stream);

/* Causal prefill that continues from an existing state (a prompt continued
 * in pieces, or chunked prefill): "恒定计算成本的工程实现" folds every token into
 * the fixed-size state, so the tokens before this call enter only through
 * S_0, the state after them (as written by sata_prefill, sata_prefill_continue
 * or sata_decode_step).  Same arguments and layouts as sata_prefill, except
 * that `state` is read as S_0 and then overwritten with the state after these
 * N tokens; out_i = (phi(q_i)^T (S_0 + sum_{j<=i} phi(k_j)[v_j,1]^T)) read
 * and normalised as in sata_prefill (j over this call's tokens, inclusive).
 * With S_0 = 0 the result equals sata_prefill's; prefill of N_0 tokens then
 * continuing with N_1 tokens gives the outputs of tokens N_0.. and the state
 * of one prefill of N_0 + N_1 tokens, up to rounding (on the tensor-core path
 * S_0 enters the readout rounded to bf16, like every chunk-boundary state).
 * Returns SATA_OK, SATA_ERR_INVALID_ARG, SATA_ERR_UNSUPPORTED, SATA_ERR_NOMEM
 * or SATA_ERR_CUDA. */
int sata_prefill_continue(const void *q, const void *k, const void *v,
                          float *out, float *state, int B, int H, int N,
                          int dK, int dV, int P, sata_dtype dt,
                          sata_stream_t stream);

/* One single-token step for each of B*H heads ("恒定计算成本的工程实现":
 * per-token procedure at constant cost): state += phi(k) [v, 1]^T in place,
 * then out = (phi(q)^T state)[:dV] / (phi(q)^T state)[dV].  The token attends
 * to itself and to everything folded into state.
 * q, k [B, H, dK]; v [B, H, dV] (dtype dt); state [B, H, m, dV+1] float,
 * updated in place; out [B, H, dV] float.
 * Returns SATA_OK, SATA_ERR_INVALID_ARG, SATA_ERR_UNSUPPORTED, SATA_ERR_NOMEM
 * or SATA_ERR_CUDA. */
int sata_decode_step(const void *q, const void *k, const void *v, float *state,
                     float *out, int B, int H, int dK, int dV, int P,
                     sata_dtype dt, sata_stream_t stream);

/* Backward pass: the gradients of L = sum(dout * out) with respect to q, k
 * and v, where out is sata_prefill's output for the same q, k, v, P
 * ("对称感知泰勒近似实现恒定Token成本注意力机制", FAQ 5: models are trained from
 * scratch with the method).  With T_ij = T_P(s_ij) on j <= i,
 *   dnum_i = dout_i / den_i, dden_i = -(dout_i . out_i) / den_i,
 *   ds_ij = (dnum_i . v_j + dden_i) T_{P-1}(s_ij),
 *   dq_i = sum_{j<=i} ds_ij k_j / sqrt(dK), dk_j = sum_{i>=j} ds_ij q_i / sqrt(dK),
 *   dv_j = sum_{i>=j} T_ij dnum_i,
 * evaluated over (query, key) tiles in fp32 on CUDA cores: exact up to
 * rounding, with a cost quadratic in N (the forward's constant-cost state is
 * not used).  q, k [B,H,N,dK] and v [B,H,N,dV] in dtype dt; dout
 * [B,H,N,dV], dq, dk [B,H,N,dK] and dv [B,H,N,dV] float; outputs must not
 * overlap each other or the inputs.  Supports every (dK, dV, P) of
 * sata_prefill.  Uses the library workspace (B*H*N*(dV+1) floats).
 * Returns SATA_OK, SATA_ERR_INVALID_ARG, SATA_ERR_UNSUPPORTED, SATA_ERR_NOMEM
 * or SATA_ERR_CUDA. */
int sata_attention_backward(const void *q, const void *k, const void *v,
                            const float *dout, float *dq, float *dk, float *dv,
                            int B, int H, int N, int dK, int dV, int P,
                            sata_dtype dt, sata_stream_t stream);

/* ---- Mixed-precision decode state ("硬件优化路径与当前局限": fp16 storage
 * halves the state's bandwidth).  The state of every head is stored as two
 * arrays: its first m_lo rows (every row of degree <= 2, m_lo =
 * C(dK+2, 2) when P >= 3, else all m rows) in fp32, and the other
 * m - m_lo rows (degree >= 3) in IEEE fp16:
 *     state_lo  [B, H, m_lo,     dV+1]  float
 *     state_hi  [B, H, m - m_lo, dV+1]  IEEE binary16 (uint16 storage)
 * Row order inside each array is the fp32 state's (degree-major,
 * lexicographic).  The low-degree rows keep fp32 because their entries grow
 * with every token (row 0 counts the tokens): in fp16 their increments would
 * be lost.  The higher-degree rows are rounded to nearest at every update. */

/* Rows per head kept in fp32 (m_lo above), or -1 if dK < 1 or P < 1.
 * Host only. */
int64_t sata_state_fp32_rows(int dK, int P);

/* Converts an fp32 state [B, H, m, dV+1] into the two arrays of the mixed
 * state (fp16 rows rounded to nearest).  state_hi may be NULL when m_lo = m.
 * Asynchronous on `stream`.  Returns SATA_OK, SATA_ERR_INVALID_ARG (null or
 * misaligned pointer, overlapping arrays, bad size), SATA_ERR_UNSUPPORTED or
 * SATA_ERR_CUDA. */
int sata_state_split(const float *state, float *state_lo, void *state_hi,
                     int B, int H, int dK, int dV, int P, sata_stream_t stream);

/* The inverse: the two arrays back into one fp32 state (exact).  Same
 * arguments and returns as sata_state_split. */
int sata_state_join(const float *state_lo, const void *state_hi, float *state,
                    int B, int H, int dK, int dV, int P, sata_stream_t stream);

/* sata_decode_step on a mixed-precision state, updated in place: the same
 * per-token procedure ("恒定计算成本的工程实现"), with each updated fp16
 * entry rounded to nearest before it is stored and read out.  dV must be 32
 * or 64 (else SATA_ERR_UNSUPPORTED); other arguments and layouts as
 * sata_decode_step.  Returns SATA_OK, SATA_ERR_INVALID_ARG,
 * SATA_ERR_UNSUPPORTED, SATA_ERR_NOMEM or SATA_ERR_CUDA; a device-side wait
 * that gave up (reported by sata_get_error as SATA_ERR_TIMEOUT) leaves the
 * state undefined. */
int sata_decode_step_mixed(const void *q, const void *k, const void *v,
                           float *state_lo, void *state_hi, float *out,
                           int B, int H, int dK, int dV, int P, sata_dtype dt,
                           sata_stream_t stream);

/* sata_decode_step without any device allocation.  (The paper has no
 * counterpart: this is an interface for callers that cannot allocate device
 * memory: hosts whose caching allocator owns the whole GPU, serving loops
 * that must not hit cudaMalloc/cudaFree because those can synchronise the
 * device, plug-in hosts whose policy forbids library-side allocations.)
 * Same arguments, layouts, semantics and results as sata_decode_step, for
 * P <= 4 (its static tables hold degrees 0..3; P = 5 -> SATA_ERR_UNSUPPORTED).  It
 * calls no cudaMalloc, cudaFree or other allocating routine: its scratch (the
 * per-head partial sums) is a file-scope __device__ array of
 * SATA_NOALLOC_MAX_PARTIALS floats (256 KiB), and its basis tables are static
 * __device__ arrays as well; every GPU that loads the library holds both
 * until the process exits.
 *   - B*H*(dV+1) > SATA_NOALLOC_MAX_PARTIALS (e.g. more than 1008 heads at
 *     dV = 64) -> SATA_ERR_INVALID_ARG, nothing launched.
 *   - The first call on a device does a one-time set-up with that device
 *     current: it resolves the arrays' device addresses with
 *     cudaGetSymbolAddress, copies the basis tables in and waits for the
 *     device (cudaDeviceSynchronize), so the tables are complete for a first
 *     call on any stream; make that first call before any stream capture.
 *   - Unlike the other calls it does not take the library's call lock.
 *   - All calls on a device share the scratch, which keeps the last call's
 *     contents; each call clears what it uses first.  Calls that overlap on
 *     the GPU (other streams or host threads) race on it: order them. */
#define SATA_NOALLOC_MAX_PARTIALS 65536
int sata_decode_step_noalloc(const void *q, const void *k, const void *v,
                             float *state, float *out, int B, int H, int dK,
                             int dV, int P, sata_dtype dt,
                             sata_stream_t stream);

/* Test hook (no counterpart on the pages).  Bounds every wait of a role in
 * the tensor-core prefill kernels and the bulk-copy decode kernel (a producer, the MMA issuer, an epilogue or
 * generator warp waiting for another role) to `cycles` SM clock cycles;
 * cycles <= 0 restores the default bound (about 2 s).  A wait that runs out
 * records SATA_ERR_TIMEOUT for sata_get_error, makes every role of its CTA
 * leave its loop, and the CTA still waits (with the default bound) for its
 * own copies and MMAs in flight and frees its TMEM before it exits; the
 * call's outputs are then incomplete.  Used by the tests to exercise that
 * path.  Returns the previous setting.  Host only. */
long long sata_test_set_wait_limit(long long cycles);

/* Synchronises `stream`, then reports (and clears) the first device-side error
 * recorded by this library's kernels on the current device (a bounded wait
 * that gave up -> SATA_ERR_TIMEOUT) or a pending CUDA error (-> SATA_ERR_CUDA).
 * Returns SATA_OK when there is none. */
int sata_get_error(sata_stream_t stream);

/* Static string for a status code (never NULL). Host only. */
const char *sata_status_string(int status);

/* Measurement hook (no counterpart on the pages; used by the benchmark).
 * sata_profile_enable(1) makes every later prefill/decode call record a pair
 * of CUDA events on its stream around each kernel it launches;
 * sata_profile_enable(0) stops it (the default).  Returns the previous
 * setting.  Host only. */
int sata_profile_enable(int on);

/* Synchronises on the events of the most recent profiled call and writes, for
 * each kernel that call launched (in launch order, at most cap), its duration
 * in milliseconds to ms_out[i] and its kernel id to ids_out[i] (either pointer
 * may be NULL).  Returns the number of kernels the call launched (may exceed
 * cap), or -1 on a CUDA error. */
int sata_profile_read(float *ms_out, int *ids_out, int cap);

/* Static name of a kernel id reported by sata_profile_read (never NULL). */
const char *sata_kernel_name(int id);

/* Frees the library's device tables and workspace on every device it touched.
 * The caller must make sure no library work is still in flight. */
void sata_release(void);

#ifdef __cplusplus
}
#endif

#endif /* SATA_H_ */
