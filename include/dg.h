/*
 * dg.h -- C ABI of the B200 (sm_100a) FP8 block-scaled GEMM library.
 *
 * The library computes D = A * B^T with A and B in FP8 E4M3 ("fn" variant,
 * max 448), fine-grained power-of-two FP32 scales, FP32 accumulation and a
 * BF16 output, in three forms:
 *
 *   dense                 D[M,N]        = A[M,K] B[N,K]^T
 *   M-grouped contiguous  D[r,:]        = A[r,:] B[m_indices[r]]^T  for every row r
 *   M-grouped masked      D[g,m,:]      = A[g,m,:] B[g]^T           for m < masked_m[g]
 *
 * and the same three forms on BF16 operands without scales (dg_bf16_*).
 *
 * Sources: the operation and its fine-grained scaling and FP32 promotion are
 * described in the DeepGEMM release article (deepseek.csdn.net), part 1.2
 * "precision safeguards"; the call names fp8_gemm_nt and
 * m_grouped_fp8_gemm_nt_contiguous in the DeepGEMM project card
 * (aiproducthub.cn), sections "quick start" and "technical implementation"
 * (M-axis grouping with N and K fixed, contiguous layout); the masked grouped
 * call (m_grouped_gemm_fp8_masked) and set_num_sms in the release article,
 * part 4.2 "advanced tuning"; the dense + contiguous + masked set in the
 * youleyou.com article "DeepGEMM -- an efficient FP8 GEMM library", section
 * on performance.
 *
 * Conventions shared by every GEMM entry point
 * --------------------------------------------
 *  - Every pointer argument is a DEVICE pointer into memory owned by the
 *    caller.  The library never frees, retains or reallocates it.
 *  - Operands (row-major, densely packed, no strides):
 *      a    E4M3 bytes, K contiguous ("K-major");
 *      b    E4M3 bytes [.., N, K], K contiguous;
 *      sfa  float32 [rows of A, K/128]: scale of A row r for K block kb is
 *           sfa[r * (K/128) + kb];
 *      sfb  float32 [.., ceil(N/128), K/128]: scale of the 128 x 128 block
 *           (n/128, kb) of B;
 *      d    bfloat16 [rows of A, N], overwritten (no C / beta input).
 *    The scales must be positive normal powers of two (2^-126 .. 2^127), as
 *    produced by scale = 2^ceil(log2(amax/448)); the kernel uses the exponent
 *    field only.  With dg_set_check_scales(1) (or DG_CHECK_SCALES=1 in the
 *    environment) the kernels check every scale they read and record device
 *    error 0x301 for one that breaks this rule (the result is then
 *    undefined); the check is off by default.
 *  - Requirements (checked on the host, DG_ERR_INVALID_ARG otherwise):
 *    K > 0 and K % 128 == 0 (BF16 operands: K % 64 == 0); N > 0 and N % 16 == 0; a, b and d 16-byte
 *    aligned, sfa/sfb 4-byte aligned, m_indices/masked_m 4-byte aligned.
 *    A zero-row problem (M == 0, M_sum == 0, G == 0 or max_m == 0) is a
 *    no-op returning DG_OK.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and return once the work is enqueued.  The device the
 *    pointers live on must be the calling thread's current CUDA device.
 *  - Errors: argument errors return before anything is launched; launch
 *    errors return DG_ERR_CUDA.  A kernel that finds an inconsistency on the
 *    device records a code that dg_get_last_device_error() reports after the
 *    stream is synchronised: 0x101..0x104 a wait that ran out of time (TMA
 *    producer, scale producer, MMA issuer, epilogue; the kernel then stops
 *    early and D is partly written), 0x201 an m_indices block naming two
 *    experts, 0x202 an expert index >= G, 0x203 K-grouped group sizes that
 *    do not tile K in multiples of 128, 0x301 a scale that is not a
 *    positive normal power of two (only when the check is on).
 *  - Results are deterministic: the same inputs give bit-identical outputs
 *    on every run (no floating-point atomics; split-K partial sums are added
 *    in a fixed order).
 *  - Thread-safe: the per-device caches are guarded by a mutex.  No call
 *    uses global scratch memory beyond the device error word, so calls may
 *    run concurrently on different streams.
 */
#ifndef DG_H_
#define DG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dg_stream_t; /* identical to cudaStream_t */

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,    /* bad size, null or misaligned pointer */
  DG_ERR_UNSUPPORTED = 2,    /* legal but not supported (e.g. too many groups) */
  DG_ERR_CUDA = 3,           /* a CUDA runtime / driver call failed */
  DG_ERR_ARCH = 4,           /* the current device is not sm_100 */
  DG_ERR_DEVICE = 5          /* a device-side error was recorded (see below) */
} dg_status;

/* Dense NT GEMM: D[M,N] = A[M,K] * B[N,K]^T.
 * a [M,K] E4M3, sfa [M, K/128], b [N,K] E4M3, sfb [ceil(N/128), K/128],
 * d [M,N] BF16.  M >= 0.
 * Usually one kernel launch on `stream`.  When the last wave of output tiles
 * would occupy at most half of the SMs (and K >= 4096), the call enqueues the
 * whole waves as one launch and the remaining tiles, one or two rectangles of
 * D, as up to two more launches of split-K tiles; dg_query_config reports the
 * split, and DG_NO_TAIL_SPLIT=1 in the environment turns it off.  The same
 * holds for dg_bf16_gemm_nt (K >= 2048 there) and dg_fp8_gemm_nt_noalloc. */
dg_status dg_fp8_gemm_nt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream);

/* The dense GEMM with other operand layouts (DeepGEMM project card,
 * aiproducthub.cn, "core features": NT / TN / NN / TT layouts on SM100).  The
 * first letter is A's layout, the second B's; "n" for A and "t" for B are
 * the K-major layouts of dg_fp8_gemm_nt:
 *   nn: a [M,K] (K-major),  b [K,N] (N-major: the element of row n and
 *       column k of B at b[k*N + n])
 *   tn: a [K,M] (M-major: a[k*M + m]),  b [K,N] (N-major)
 *   tt: a [K,M] (M-major),  b [N,K] (K-major)
 * D[M,N] = A * B^T in every case, with the scales, D and all other rules of
 * dg_fp8_gemm_nt (sfa [M, K/128], sfb [ceil(N/128), K/128], d [M,N] BF16).
 * An M-major A needs M % 16 == 0 (its rows of M bytes are 16-byte units);
 * otherwise DG_ERR_INVALID_ARG. */
dg_status dg_fp8_gemm_nn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream);
dg_status dg_fp8_gemm_tn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream);
dg_status dg_fp8_gemm_tt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream);

/* Dense NT GEMM with FP32 output and an optional FP32 addend (the `c`
 * argument of the DeepGEMM project card's "quick start" call
 * fp8_gemm_nt(a, b, c, a_sf, b_sf)):
 *   D[M,N] = A[M,K] * B[N,K]^T + C[M,N]     (C == NULL: D = A * B^T)
 * a, sfa, b, sfb as in dg_fp8_gemm_nt; c and d float32 [M,N], row-major,
 * 16-byte aligned; c may equal d (accumulate in place).  The FP32
 * accumulator is added to C and stored without rounding to BF16. */
dg_status dg_fp8_gemm_nt_f32(const void* a, const float* sfa, const void* b, const float* sfb,
                             const float* c, float* d, int M, int N, int K, dg_stream_t stream);

/* M-grouped GEMM, contiguous layout (MoE experts' tokens concatenated along M).
 * a [M_sum,K], sfa [M_sum,K/128], b [G,N,K], sfb [G,ceil(N/128),K/128],
 * d [M_sum,N], m_indices int32 [M_sum] (device): the expert of row r, or -1
 * for a padding row, whose row of D is left untouched.  M_sum % 128 == 0, and
 * every aligned block of 128 rows holds rows of at most one expert (plus
 * padding): each expert's segment starts at a multiple of 128.  Rows whose
 * index is another expert than their block's, or >= G, are not written and
 * set a device error. */
dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, void* d, const int* m_indices,
                                              int M_sum, int N, int K, int G, dg_stream_t stream);

/* M-grouped GEMM, masked layout (decode: token counts known only on the device).
 * a [G,max_m,K], sfa [G,max_m,K/128], b [G,N,K], sfb [G,ceil(N/128),K/128],
 * d [G,max_m,N], masked_m int32 [G] (device): rows m >= masked_m[g] of group g
 * (clamped to [0, max_m]) are never written.  expected_m is a host-side hint
 * of the typical masked_m used only to pick a configuration; results do not
 * depend on it.  G <= 1024. */
dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const float* sfa, const void* b,
                                          const float* sfb, void* d, const int* masked_m, int G,
                                          int max_m, int N, int K, int expected_m,
                                          dg_stream_t stream);

/* K-grouped GEMM, contiguous layout: the weight gradient of the M-grouped
 * forms in training (DeepGEMM project card, aiproducthub.cn, "core
 * features": the unified GEMM family serves training forward and backward,
 * with NT / TN / NN / TT layouts on SM100).  The tokens of all G groups
 * (experts) are concatenated along the reduction axis K; group g owns the K
 * rows [k_off[g], k_off[g] + ks[g]) with k_off[g] = ks[0] + ... + ks[g-1]:
 *   D[g][M,N] = C[g] + sum over the K rows k of group g of A_hat[k,:]^T B_hat[k,:]
 * a    E4M3 bytes [K_sum, M], M contiguous (M-major: one row per token);
 * b    E4M3 bytes [K_sum, N], N contiguous (N-major);
 * sfa  float32 [M, K_sum/128]: scale of output row m for the K block kb
 *      (the global block index: k / 128);
 * sfb  float32 [ceil(N/128), K_sum/128]: scale of the 128 x 128 block
 *      (n/128, kb) of B;
 * c, d float32 [G, M, N]; c may be NULL (D = the products) or equal d
 *      (accumulate in place, as a training step does);
 * ks   int32 [G] on the device: every ks[g] >= 0, a multiple of 128 (each
 *      group's token segment padded to 128 rows, so no scale block spans two
 *      groups), summing to K_sum.  A group with ks[g] == 0 gets D[g] = C[g]
 *      (zeros without C).  Sizes that break these rules are found on the
 *      device: nothing is written and device error 0x203 is recorded.
 * M % 16 == 0 (M-major rows of whole 16-byte units), N % 16 == 0,
 * K_sum > 0 and K_sum % 128 == 0, G <= 1024, a, b, c, d 16-byte aligned;
 * otherwise DG_ERR_INVALID_ARG (DG_ERR_UNSUPPORTED for G > 1024).  The scale
 * contract and everything else are those of the dense calls. */
dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, const float* c, float* d,
                                              const int* ks, int G, int M, int N, int K_sum,
                                              dg_stream_t stream);

/* The three GEMM forms on BF16 operands (DeepGEMM project card,
 * aiproducthub.cn, "core features": BF16 beside FP8 and FP4 in the unified
 * dense GEMM family; grouped GEMMs in contiguous and masked layouts for MoE).
 * No scale factors: D = bf16(A * B^T), FP32 accumulation, one rounding.
 * a and b hold BF16 elements (2 bytes), both K-major; d is BF16; K % 64 == 0
 * (one 128-byte K block is 64 elements).  Shapes, m_indices, masked_m,
 * expected_m, untouched rows and every other rule are those of the FP8
 * functions with the same form:
 *   dense:      a [M,K], b [N,K], d [M,N]
 *   contiguous: a [M_sum,K], b [G,N,K], d [M_sum,N], m_indices [M_sum]
 *   masked:     a [G,max_m,K], b [G,N,K], d [G,max_m,N], masked_m [G] */
dg_status dg_bf16_gemm_nt(const void* a, const void* b, void* d, int M, int N, int K,
                          dg_stream_t stream);
dg_status dg_m_grouped_bf16_gemm_nt_contiguous(const void* a, const void* b, void* d,
                                               const int* m_indices, int M_sum, int N, int K,
                                               int G, dg_stream_t stream);
dg_status dg_m_grouped_bf16_gemm_nt_masked(const void* a, const void* b, void* d,
                                           const int* masked_m, int G, int max_m, int N, int K,
                                           int expected_m, dg_stream_t stream);

/* Cap on the number of SMs the GEMMs use (release article, part 4.2:
 * set_num_sms).  n <= 0 restores the default (all SMs of the device).
 * Applies to later calls from every thread. */
dg_status dg_set_num_sms(int n);
/* The cap in force for the current device (its SM count when no cap is set),
 * or -1 if no CUDA device is usable. */
int dg_get_num_sms(void);

/* Reads and clears the device error word of the current device.  *code is 0
 * when no device-side error was recorded since the last call.  Synchronises
 * the device.  Returns DG_ERR_CUDA if the device cannot be queried. */
dg_status dg_get_last_device_error(int* code);

/* Per-launch time limit of every wait inside the kernels, in milliseconds
 * (default 1000, or DG_WAIT_TIMEOUT_MS from the environment).  A wait that
 * runs out records a device error (0x101..0x104) and the kernel returns
 * instead of hanging.  Applies to launches enqueued after the call, from
 * every thread and entry point.  ms <= 0: DG_ERR_INVALID_ARG. */
dg_status dg_set_wait_timeout_ms(int ms);
/* The same limit in nanoseconds, for limits shorter than a millisecond (a
 * wait needs at least one poll of the GPU's global timer, whose ticks are
 * tens to hundreds of nanoseconds apart, before it can run out). */
dg_status dg_set_wait_timeout_ns(long long ns);

/* Turns the kernels' check of the scale contract on (enable != 0) or off:
 * every scale a kernel reads must be a positive normal power of two, and one
 * that is not records device error 0x301.  Off by default; the environment
 * variable DG_CHECK_SCALES=1 turns it on at first use.  Applies to launches
 * enqueued after the call, from every thread and entry point.  When on, each
 * FP8 call first launches a small kernel on the same stream that reads every
 * scale of sfa and sfb (one extra launch per call); when off, nothing is
 * added. */
dg_status dg_set_check_scales(int enable);

/* Weight preload for the dense calls (enable != 0), off by default; the
 * environment variable DG_WEIGHT_PRELOAD=1 turns it on at first use.  Every
 * GEMM launch may start before the previous kernel on its stream has
 * finished (programmatic dependent launch) and waits for it before reading
 * its inputs.  With the preload on, a dense call's kernel loads the first
 * ring stages of B before that wait, overlapping them with the previous
 * kernel's tail; only A (and the scales) are read after it.  The caller
 * declares by turning it on that B -- model weights in inference -- is
 * never written by a kernel that may still run when a dense GEMM reading it
 * is launched on the same stream.  Applies to launches enqueued after the
 * call, from every thread and entry point; results are the same either way
 * when that holds. */
dg_status dg_set_weight_preload(int enable);

/* Human-readable name of a status code.  Never NULL. */
const char* dg_status_string(dg_status s);

/* Configuration the picker chooses for a problem, without launching anything
 * and without a GPU (num_sms is given explicitly).  kind: 0 dense, 1
 * contiguous, 2 masked, 3 K-grouped; rows: M, M_sum or max_m (K-grouped: M,
 * the output rows of each group; K: K_sum); expected_m only for masked.
 * The picker counts K in 128-byte blocks of a row: for the BF16-operand
 * calls pass 2 * K (their tile geometry is that of the E4M3 call with twice
 * the K, without the scale factors' shared memory and TMEM columns).
 * For the masked form the grid is an upper bound (the real tile count is
 * read from masked_m on the device). */
typedef struct {
  int block_m;     /* rows of A per tile (128) */
  int block_n;     /* rows of B (columns of D) per tile */
  int stages;      /* depth of the shared-memory operand ring */
  int num_acc;     /* TMEM accumulator buffers */
  int split_k;     /* K slices per output tile (> 1: one CTA cluster per tile) */
  int grid;        /* CTAs launched */
  int smem_bytes;  /* dynamic shared memory per CTA */
  int tmem_cols;   /* TMEM columns allocated per CTA */
  int kps;         /* 128-wide K blocks per ring stage */
  int main_tiles;  /* dense form: tiles of the first launch when the last wave
                      is split off (0: one launch) */
  int tail_launches; /* launches of 128 x 128 decode tiles after the first (0..2):
                        the tiles past main_tiles, one rectangle of D each */
  int tail_split;  /* K slices (CTAs per cluster) of the tail launches' tiles */
} dg_config;

dg_status dg_query_config(int kind, int rows, int N, int K, int G, int expected_m, int num_sms,
                          dg_config* out);

/* Dense NT GEMM that allocates no device memory, for callers that cannot call
 * cudaMalloc -- e.g. code running under a caching allocator or a memory pool
 * that owns all device memory, or a host that must not grow its footprint
 * after start-up.  The pages have no counterpart of this call.
 *
 * Same operands, layouts and requirements as dg_fp8_gemm_nt.  The only
 * scratch it needs, the device error word that the kernel's bounded waits
 * report into, is a fixed 256-byte __device__ array inside the library,
 * which every GPU that loads the library holds until the process exits
 * (split-K partial sums stay in on-chip shared memory, so no problem size
 * needs more).  It calls no cudaMalloc, cudaFree or allocating library
 * routine.
 *
 * The first call on a device sets that device up (architecture check,
 * cluster-occupancy query and the device address of the array through
 * cudaGetSymbolAddress); make that first call before any stream capture.
 * Every call shares the one array, which keeps the last call's contents;
 * calls whose kernels overlap on the GPU (different streams, or several
 * threads) share it too.  The SM cap of dg_set_num_sms does not apply here
 * (all SMs are used).  Waits inside the kernel are bounded by the same limit
 * as every call (dg_set_wait_timeout_ms / _ns), and DG_NO_PREFETCH and
 * DG_CHECK_SCALES apply as they do elsewhere.  Device-side error codes of
 * this call go to the array's error word, not to the one
 * dg_get_last_device_error reads: read them with
 * dg_fp8_gemm_nt_noalloc_get_last_device_error. */
dg_status dg_fp8_gemm_nt_noalloc(const void* a, const float* sfa, const void* b,
                                 const float* sfb, void* d, int M, int N, int K,
                                 dg_stream_t stream);

/* Reads and clears the error word of dg_fp8_gemm_nt_noalloc on the current
 * device (codes as for dg_get_last_device_error; 0: none since the last
 * read).  Synchronises the device, then copies the word through the CUDA
 * symbol API, which allocates no device memory.  Since every no-alloc call
 * shares the word, a code may come from any of the calls since the last
 * read.  Returns DG_ERR_CUDA if the device cannot be queried. */
dg_status dg_fp8_gemm_nt_noalloc_get_last_device_error(int* code);

/* Library version, "major.minor.patch". */
const char* dg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
