/*
 * lwq.h -- block-quantized matmul for NVIDIA B200 (sm_100a).
 *
 *     y[M,N] = x[M,K] . dequant(Wq[N,K])^T
 *
 * The weights Wq are stored in llama.cpp-style blocks (the "legacy" and
 * "K-quant" families named in "Resumo Tecnico: Llamas na Web",
 * "Declaracao do Problema" item 3, and in its "3. Design de Shader Consciente
 * de Quantizacao", which co-designs dequantization with the matmul kernels:
 * decoded in registers for the matrix-vector (decode) case and in shared
 * memory, reused across rows, for the matrix-matrix (prefill) case).
 *
 * Paths (chosen per call by a per-shape configuration table, the analogue of
 * the tunable tile sizes in "2. Biblioteca de Kernels Portatil em
 * Desempenho", "Parametros Ajustaveis"):
 *   M <= 16  decode GEMV: packed rows staged by TMA into shared memory,
 *            decoded in registers, multiplied on the tensor cores with
 *            warp-level MMAs, split-K partials reduced deterministically;
 *   M >  16  prefill GEMM: packed tiles staged by TMA, dequantized to
 *            bf16/fp16 in shared memory, tcgen05 MMAs accumulating in TMEM.
 * Q6_K rows that are not 16-byte multiples (K not a multiple of 2048) and Q2_K
 * rows (K not a multiple of 1024) stream as slots of the flat matrix (whole
 * 16-byte units per row) into both paths, which needs N * lwq_row_bytes(fmt,
 * K) to be a multiple of 16.  Shapes
 * no tensor-core path takes (K not a multiple of 256, or such a matrix that is
 * not a whole number of 16-byte units) run a simple GEMV kernel.
 *
 * Everything is plain C: pointers and sizes, no C++ or framework types.
 */
#ifndef LWQ_H
#define LWQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
typedef enum {
    LWQ_OK = 0,
    LWQ_ERR_INVALID_ARG = 1,        /* a size is <= 0, K is not a multiple of the block, NULL pointer */
    LWQ_ERR_UNSUPPORTED = 2,        /* unknown format / activation code, or a shape no path handles */
    LWQ_ERR_MISALIGNED = 3,         /* Wq, x, y or the workspace is not 16-byte aligned */
    LWQ_ERR_NOT_INITIALIZED = 4,    /* a call needs the workspace and lwq_init was not called on this device */
    LWQ_ERR_WORKSPACE_TOO_SMALL = 5,/* the registered workspace is smaller than this call needs */
    LWQ_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed (launch error, bad device) */
    LWQ_ERR_DEVICE_TIMEOUT = 7      /* a kernel gave up a bounded wait (see lwq_get_device_error) */
} lwq_status;

/* ------------------------------------------------- format and dtype codes
 * fmt = weight format | activation dtype [| flags, below].
 *
 * LWQ_Q8_0: 32 weights per 34-byte block: fp16 d (little endian), int8 q[32];
 *           w = d*q.
 * LWQ_Q4_0: 32 weights per 18-byte block: fp16 d, 16 bytes b[16]; byte i
 *           holds element i in its low nibble and element i+16 in its high
 *           nibble; w = (nibble - 8)*d.
 * LWQ_Q4_K: 256 weights per 144-byte superblock: fp16 d, fp16 dmin, 12 bytes
 *           of eight 6-bit (scale, min) pairs (for j < 4: sc_j = s[j]&63,
 *           m_j = s[j+4]&63; for j >= 4: sc_j = (s[j+4]&15)|((s[j-4]>>6)<<4),
 *           m_j = (s[j+4]>>4)|((s[j]>>6)<<4)), 128 bytes of nibbles in 4
 *           groups of 32 (group g: low nibbles are sub-block 2g, high
 *           nibbles sub-block 2g+1); w = d*sc_j*q - dmin*m_j.
 * More K-quant formats of the same family ("Resumo Tecnico: Llamas na Web"
 * names q4_k_m, which mixes Q4_K and Q6_K tensors, and q2_k, without their
 * layouts; these are the llama.cpp layouts of those names):
 * LWQ_Q6_K: 256 weights per 210-byte superblock: ql[128] (low 4 bits of the
 *           6-bit codes), qh[64] (high 2 bits), int8 sc[16] (one scale per 16
 *           weights), fp16 d.  Element 128n+32g+l (n<2, g<4, l<32) takes
 *           nibble g>>1 of ql[64n+32(g&1)+l] and bits 2g, 2g+1 of qh[32n+l];
 *           w = d*sc[e/16]*(q - 32).
 * LWQ_Q5_K: 256 weights per 176-byte superblock: fp16 d, fp16 dmin, the 12
 *           scale/min bytes of Q4_K, qh[32], qs[128].  Element 64g+32h+l
 *           takes nibble h of qs[32g+l] and (as bit 4) bit 2g+h of qh[l];
 *           w = d*sc_j*q - dmin*m_j, j = 2g+h.
 * LWQ_Q2_K: 256 weights per 84-byte superblock: s[16] (per 16 weights: scale
 *           in the low nibble, min in the high nibble), qs[64], fp16 d, fp16
 *           dmin.  Element 128n+32j+l takes bits 2j, 2j+1 of qs[32n+l];
 *           w = d*(s[e/16]&15)*q - dmin*(s[e/16]>>4).
 * Activations x: fp32, fp16 or bf16, row-major [M][K].
 */
#define LWQ_Q8_0 1
#define LWQ_Q4_0 2
#define LWQ_Q4_K 3
#define LWQ_Q6_K 4
#define LWQ_Q5_K 5
#define LWQ_Q2_K 6
#define LWQ_FMT_MASK 0xFF
#define LWQ_ACT_F32 0x000
#define LWQ_ACT_F16 0x100
#define LWQ_ACT_BF16 0x200
#define LWQ_ACT_MASK 0xF00
/* Optional flag, or-ed into fmt: the caller promises that Wq is not written
 * by any work still running on the stream when the call is made (weights are
 * constant, as in a decode loop).  The call's kernels are then launched as
 * programmatic dependent launches: they may start, and begin streaming Wq,
 * before the preceding kernel on the stream has finished; they still wait for
 * it to complete before reading x or writing y and the workspace.  This hides
 * launch latency between back-to-back calls. */
#define LWQ_FLAG_OVERLAP 0x1000
/* Optional flag, or-ed into fmt: int8 activation blocks ("quantized arithmetic
 * without runtime dequantization", "Compute Shaders con WebGPU para Inferencia
 * ML").  Each run of 32 activations of a row (K must be a multiple of 256) is
 * quantized in the kernel to int8 codes q with one fp32 scale d, per block in
 * fp32 with round-to-nearest-even:
 *   amax = max |x|;  amax < 2^-100: d = 0, q = 0;  else d = amax / 127,
 *   q = rint(x * (127 / amax)),
 * 16-bit activations first widened exactly; and y = x_q * dequant(Wq)^T with
 * x_q = q * d, the block dot products taken in integers (s8 x s8 -> s32) and
 * scaled in fp32.  Results differ from the unquantized product by the
 * activation rounding (max |y - y_exact| / sum |x w| stays below 1e-2 for
 * N(0,1) activations); against x_q they agree to fp32 rounding.  Supported for
 * Q4_0, Q8_0 and Q4_K weights at any M, in passes of 8 activation rows (each pass
 * streams the weights: a prefill-sized M reads them M/8 times); other formats
 * return LWQ_ERR_UNSUPPORTED.  Activations must be finite. */
#define LWQ_FLAG_ACT_I8 0x2000

/* Bytes of one packed row of K weights (K/32*34, K/32*18, K/256*144,
 * K/256*210, K/256*176, K/256*84), or 0
 * when fmt is unknown or K is not a positive multiple of the block size. */
size_t lwq_row_bytes(int fmt, int64_t K);

/* Device workspace bytes that lwq_matmul needs for every call with
 * M <= max_M, N <= max_N, K <= max_K in this format.  The workspace holds the
 * split-K partial sums (fp32), which a follow-up kernel adds in split order
 * (deterministic); it is the library's one static arena,
 * sized once at start-up ("1. Inferencia Local Eficiente em Memoria",
 * "Alocacao Estatica de Memoria" and "Arena de Buffer de Parametros").
 * Returns 0 for invalid arguments. */
size_t lwq_workspace_size(int fmt, int max_M, int max_N, int max_K);

/* Register the caller-owned device workspace for the CURRENT device.
 * d_workspace: device pointer, 16-byte aligned (NULL with bytes == 0 is
 * allowed: calls that need no workspace still run).  The library keeps the
 * pointer until lwq_shutdown or the next lwq_init on this device; it never
 * allocates, frees or reads it outside lwq_matmul, and its contents need no
 * initial value.  No device work is done here.  Errors: LWQ_ERR_MISALIGNED,
 * LWQ_ERR_INVALID_ARG, LWQ_ERR_CUDA (no current device). */
int lwq_init(void *d_workspace, size_t bytes);

/* Forget the workspace registered for the current device.  Always LWQ_OK. */
int lwq_shutdown(void);

/*
 * y[M,N] (fp32, row-major) = x[M,K] . dequant(Wq)^T.
 *
 *   fmt     weight format | activation dtype, optionally | LWQ_FLAG_OVERLAP
 *           and | LWQ_FLAG_ACT_I8 (codes above)
 *   Wq      device pointer, N packed rows of lwq_row_bytes(fmt, K) bytes each
 *   x       device pointer, row-major [M][K] in the activation dtype
 *   y       device pointer, row-major [M][N] fp32, fully overwritten
 *   M, N, K sizes (> 0); K a multiple of 32 (Q8_0, Q4_0) or 256 (K-quants)
 *   stream  a cudaStream_t (NULL = the legacy default stream)
 *
 * Ownership: the caller owns Wq, x, y and the workspace.  The call is
 * asynchronous: it validates the arguments on the host, enqueues its
 * kernels on `stream` (one per pass of activation rows, plus a split-K sum
 * kernel per pass when K is split; lwq_last_launch_count tells how many) and
 * returns; it never allocates and never synchronizes
 * the host.  Kernel faults surface at the caller's next synchronization, as
 * with any CUDA launch.  Wq, x and y must be 16-byte aligned
 * (LWQ_ERR_MISALIGNED).  Calls that use split-K (see lwq_workspace_size) need
 * a registered workspace (LWQ_ERR_NOT_INITIALIZED,
 * LWQ_ERR_WORKSPACE_TOO_SMALL); calls sharing one workspace must be ordered
 * (one stream, or events), since their partial sums share the arena.  A GEMV
 * call whose chosen plan splits K but finds too little workspace takes the
 * plan with a warp per chunk of K instead when that one needs no more (the
 * K-quants with 9..16 rows of 16-bit x or 3..5 of fp32 x and K <= 4096), so it
 * runs as it would with no workspace; lwq_workspace_size covers the faster plan.
 * M > 16 with fp32 activations runs the GEMV path over groups of rows of x.
 */
int lwq_matmul(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, void *stream);

/* lwq_matmul for callers that cannot allocate device memory: code that may
 * not call the CUDA allocator (an allocator's own callbacks, a process whose
 * memory pool is fixed and fully handed out at start-up, a plugin given only
 * input and output pointers).  It needs no workspace and no lwq_init: its
 * split-K scratch is a static 4 MiB device array inside the library, held on
 * every device that loads the library until the process exits.  The pages
 * this library follows have no counterpart of this entry point.
 *
 * Arguments, layouts and results are those of lwq_matmul.  Only the decode
 * GEMV is offered: M <= 16 and the shapes lwq_select_config sends to path 1,
 * else LWQ_ERR_UNSUPPORTED.  A shape whose split-K scratch
 * (lwq_workspace_size bytes) exceeds 4 MiB returns LWQ_ERR_WORKSPACE_TOO_SMALL.
 * The first call on a device looks up the array's device address (make it
 * before any stream capture).  Calls share the array, which needs no initial
 * value; calls whose kernels overlap on the GPU race.  Nothing is allocated
 * or freed. */
int lwq_matmul_noalloc(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, void *stream);

/* ------------------------------------------------ configuration table
 * The per-shape configuration lwq_matmul would use, and a way to force one
 * (used by the sweep that fills the table and by tests). */
typedef struct {
    int path;        /* 1 = GEMV (tensor-core MMA), 2 = GEMM (tcgen05), 3 = simple GEMV */
    int warps;       /* GEMV: compute warps per CTA, each owning 256 weights of K */
    int stages;      /* pipeline depth (shared-memory ring stages) */
    int splits;      /* GEMV: split-K factor (1 = none) */
    int ctas;        /* CTAs launched (persistent grid) */
    int tile_n;      /* GEMM: output columns per tile (weight rows): 128, or 256 as two
                        128-row halves sharing each activation tile */
    int tile_m;      /* GEMM: output rows per tile (activation rows) */
    int reserved[5];
} lwq_config;

/* Fill *cfg with the configuration lwq_matmul(fmt, ., ., ., M, N, K) would
 * use on the current device.  Errors as lwq_matmul's argument checks. */
int lwq_select_config(int fmt, int M, int N, int K, lwq_config *cfg);

/* lwq_matmul with a forced configuration.  Fields set to 0 take the table's
 * value; an impossible configuration returns LWQ_ERR_UNSUPPORTED. */
int lwq_matmul_config(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K,
                      const lwq_config *cfg, void *stream);

/* ------------------------------------------------------ decode attention
 * One query token per sequence and head against that sequence's key/value
 * cache, the softmax fused into the one pass over the keys ("Compute Shaders
 * con WebGPU para Inferencia ML", "El Mecanismo de Atencion": scores
 * q.k / sqrt(head_dim), a running maximum and sum, the weighted values
 * accumulated in the same pass):
 *   s_j = scale * (q . k_j),  out = sum_{j < len} softmax(s)_j v_j.
 * dtype: LWQ_ACT_F16 or LWQ_ACT_BF16, the type of q, k and v.
 * q [B][H][D]; k, v [B][Hkv][Lmax][D] (the caches, key j of sequence b and kv
 * head g at [b][g][j]); out [B][H][D] fp32; all row-major device arrays,
 * 16-byte aligned.  Query head h reads kv head h / (H / Hkv); H / Hkv must be
 * 1, 2, 4 or 8, and D 64 or 128.  seq_lens: device array of B int32 lengths
 * (a length outside [1, Lmax] is clamped into it), or NULL for Lmax each.
 * scale: usually 1 / sqrt(D).  Long sequences are split over several CTAs
 * whose partial results a second kernel merges; the partials live in the
 * workspace registered with lwq_init (the static arena that "Llamas na Web",
 * "Alocacao Estatica de Memoria", sizes at start-up for FlashAttention-style
 * scratch), lwq_attention_workspace_size bytes.  Errors: LWQ_ERR_INVALID_ARG
 * (a size <= 0, H not a multiple of Hkv, NULL q/k/v/out, non-finite scale),
 * LWQ_ERR_UNSUPPORTED (dtype, D, H / Hkv), LWQ_ERR_MISALIGNED,
 * LWQ_ERR_NOT_INITIALIZED / LWQ_ERR_WORKSPACE_TOO_SMALL (split partials),
 * LWQ_ERR_CUDA.  The library allocates nothing and does not synchronize. */
size_t lwq_attention_workspace_size(int B, int H, int Hkv, int Lmax, int D);
int lwq_attention_decode(int dtype, const void *q, const void *k, const void *v, const int32_t *seq_lens, float *out,
                         int B, int H, int Hkv, int Lmax, int D, float scale, void *stream);

/* ------------------------------------------------ errors and diagnostics */

/* Static description of a status code. */
const char *lwq_status_string(int status);

/* Device-side error word of the current device: every wait in the kernels
 * (on an mbarrier or a TMEM handoff) is bounded, in lwq_matmul and
 * lwq_matmul_noalloc alike; a kernel
 * that gives up sets a bit here and returns instead of hanging.  The caller
 * must synchronize first.  Returns LWQ_OK, LWQ_ERR_DEVICE_TIMEOUT (and clears
 * the word), or LWQ_ERR_CUDA. */
int lwq_get_device_error(void);

/* Launch a one-CTA kernel on `stream` that waits on an mbarrier nothing ever
 * arrives at, with a wait bound of timeout_us microseconds, so that callers
 * can check that bounded waits end and report LWQ_ERR_DEVICE_TIMEOUT through
 * lwq_get_device_error.  Faults nothing and hangs nothing. */
int lwq_selftest_timeout(unsigned timeout_us, void *stream);

/* Number of kernels the last successful lwq_matmul / lwq_matmul_config call
 * on this thread enqueued. */
int lwq_last_launch_count(void);

/* Library version, e.g. 0x000100 for 0.1.0. */
int lwq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LWQ_H */
