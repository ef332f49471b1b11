/*
 * qnt.h -- C ABI of libqnt: round-to-nearest (RTN) group-wise 4-bit weight
 * quantization and decode-time fused-dequant GEMV / small-batch GEMM on one
 * NVIDIA B200 (sm_100a).
 *
 * What the operations are, by source page:
 *  - "Is (Selective) Round-To-Nearest Quantization All You Need?" (Kogan,
 *    arXiv 2505.15909), English abstract: RTN is cheap to apply, its token
 *    generation throughput with fused-dequant kernels can beat advanced
 *    methods, and accuracy improves by raising the precision of selected
 *    layers / modules -> qnt_quantize, qnt_gemv / qnt_gemm, qnt_table_*.
 *  - "Revisiting Block-based Quantisation" (Zhang et al., arXiv 2310.05079),
 *    English abstract: scaling factors shared across a block of packed numbers
 *    -> the `group` (block) size along the input dimension.
 *  - "The Power of Negative Zero: RaZeR" (Chen et al., arXiv 2501.04052),
 *    English abstract and method section: FP4 whose negative-zero code is
 *    remapped to a special value, and a fast fused-dequant GEMV -> QNT_FP4_RAZER.
 *  - "AFPQ: Asymmetric Floating Point Quantization" (Zhang et al., arXiv
 *    2311.01792), English abstract: separate scales for positive and negative
 *    values -> QNT_FP4_AFPQ.
 * The pages give no formulas; the exact arithmetic of each format is stated
 * below with each enum value.
 *
 * Conventions (all entry points):
 *  - W is [N][K] row-major (N = output features, K = input features, the
 *    PyTorch nn.Linear convention).  Groups are runs of `group` consecutive
 *    weights along K inside one row.  x is [K], y is [N]; X is [M][K] and Y
 *    is [M][N], row-major.
 *  - Every buffer argument named d_* or documented "device" is device memory
 *    that the CALLER allocates and owns.  The library never allocates or frees
 *    memory, keeps no state between calls and is safe to call from several
 *    host threads.  Work is enqueued asynchronously on `stream` (a
 *    cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - The return value is the host-side validation result.  On any error
 *    nothing is launched.  Device-detected conditions (non-finite weights,
 *    scale overflow, a bounded wait that expired) are written to the optional
 *    device int *d_status (may be NULL) with an atomic max, never cleared by
 *    the library: zero it before the call, read it after synchronizing.
 *  - Pointers to packed codes, metadata, activations and outputs must be 16-byte
 *    aligned (QNT_ERR_ALIGN otherwise).
 */
#ifndef QNT_H_
#define QNT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QNT_VERSION 3

/* Largest K that qnt_gemv, qnt_gemm and qnt_gemv_seq accept: every GEMV
 * kernel stages the activation vector (2K bytes) in shared memory next to its
 * weight ring, and the CUDA-core kernel (INT8, FP16, batch 2) would not fit at
 * K = 65536.  qnt_quantize accepts K up to 2^20. */
#define QNT_MAX_GEMV_K 32768

/* Weight formats.  h(.) = round-to-nearest-even to fp16; every quotient below
 * is one IEEE binary32 division; rint = round half to even; a scale that
 * rounds to zero is stored as 1.0; a scale that overflows fp16 sets
 * QNT_ERR_RANGE in *d_status. */
typedef enum {
  /* Asymmetric INT4 (asymmetric INT named by the RaZeR and AFPQ abstracts):
   * s = h((max - min) / 15), z = clamp(rint(-min / s), 0, 15),
   * q = clamp(rint(w / s) + z, 0, 15), dequant = (q - z) * s.
   * Metadata 2.5 bytes per group (fp16 scale, 4-bit zero). */
  QNT_INT4_ASYM = 1,
  /* Symmetric FP4 E2M1 (sign-magnitude 4-bit float of the RaZeR page): codes
   * 0..7 = 0, .5, 1, 1.5, 2, 3, 4, 6, bit 3 = sign; s = h(absmax / 6);
   * code = nearest value to w / s (ties to even mantissa, saturating at 6);
   * magnitude 0 is always code 0 (0b1000 is never produced). 2 bytes/group. */
  QNT_FP4_E2M1 = 2,
  /* AFPQ: s+ = h(max(max, 0) / 6), s- = h(max(-min, 0) / 6); positive weights
   * use s+, negative weights s- (sign bit set); dequant = e2m1(code) * s+ or
   * * s-.  4 bytes/group. */
  QNT_FP4_AFPQ = 3,
  /* RaZeR: E2M1 whose code 0b1000 decodes to a special value sv chosen per
   * group from {+5, -5, +8, -8} (2-bit selector 0..3 in that order).  For each
   * candidate: s = h(absmax / max(6, |sv|)), codes = nearest of the 15 regular
   * values and sv (a tie with sv goes to the regular value); the candidate with
   * the smallest binary64 sum of squared errors (summed as a balanced binary
   * tree in index order) wins, ties to the smaller selector.  2.25 bytes/group. */
  QNT_FP4_RAZER = 4,
  /* INT8 symmetric per output channel (selective precision): s = h(absmax_row
   * / 127), q = clamp(rint(w / s), -127, 127).  group must equal K. */
  QNT_INT8_PERCHAN = 5,
  /* FP16 (selective precision, no quantization): code = h(w).  group == K. */
  QNT_FP16 = 6
} qnt_fmt;

/* Activation / output element type.  y and Y use the activation type. */
typedef enum { QNT_F16 = 0, QNT_BF16 = 1 } qnt_dtype;

/* Error codes. */
enum {
  QNT_OK = 0,
  QNT_ERR_ARG = 1,       /* null pointer, unknown format / dtype, M out of range */
  QNT_ERR_SHAPE = 2,     /* N < 1, K % 128 != 0, group not in {32,64,128} (4-bit) or != K,
                            K > QNT_MAX_GEMV_K for a GEMV / GEMM */
  QNT_ERR_ALIGN = 3,     /* a buffer is not 16-byte aligned */
  QNT_ERR_CUDA = 4,      /* the kernel launch failed */
  QNT_ERR_TIMEOUT = 5,   /* (device) a bounded wait for an asynchronous copy expired */
  QNT_ERR_NONFINITE = 6, /* (device) NaN or Inf in W; codes are unspecified */
  QNT_ERR_RANGE = 7      /* (device) a scale or FP16 code overflowed fp16 */
};

/* Shape and format of one quantized matrix. */
typedef struct {
  int32_t fmt;    /* qnt_fmt */
  int32_t N;      /* output features (rows of W), >= 1 */
  int32_t K;      /* input features, a positive multiple of 128 */
  int32_t group;  /* 32, 64 or 128 for 4-bit formats; K for INT8 / FP16 */
} qnt_desc;

/*
 * Packed storage layout (one layout serves qnt_gemv and qnt_gemm).
 *
 * 4-bit codes: rows are stored in groups of eight.  Row group R = n/8 occupies
 * 4K bytes at byte R*4K (the buffer holds ceil(N/8)*8 rows; the contents of
 * padding rows are unspecified and never reach a result).  Within a group,
 * block b (weights 128b..128b+127 of each of its eight rows) occupies 512
 * bytes at offset 512b; row i = n%8 sits at offset 64i inside the block as four
 * 16-byte chunks, chunk c (weights 128b+32c .. 128b+32c+31 of the row) at byte
 * 64i + 16*(c XOR ((i/2) % 4)).  The 16 bytes of a chunk are four little-endian
 * 32-bit words, and nibble p (bits 4p..4p+3) of word j holds chunk weight
 *   QNT_INT4_ASYM:                 16*(p%2) + 4j + 2*((p/2)%2) + p/4
 *   QNT_FP4_E2M1 / AFPQ / RAZER:   8j + p
 * So 256 consecutive weights of eight rows are one contiguous 1 KB run (one
 * bulk copy), eight threads that read the same chunk of eight rows of a group
 * (or the four chunks of two rows) hit distinct shared-memory bank groups, and
 * the INT4 order turns a word into
 * fp16 pairs with two masks and one shift (low nibbles give chunk weights 0..15
 * in order, high nibbles 16..31).  FP4-family bytes hold two consecutive
 * weights, low nibble first.
 * INT8 codes: row-major int8 [N][K].  FP16 codes: row-major fp16 [N][K].
 *
 * Metadata buffer (byte offsets), G = K/group, P = N*G, group f = n*G + j:
 *   INT4:  fp16 scale[P] at 0; 4-bit zeros from Z0 = round_up(2P, 256):
 *          zero of group f in byte Z0 + f/2, low nibble when f is even;
 *          the zero plane is round_up(ceil(P/2), 16) bytes long.
 *   FP4:   fp16 scale[P] at 0.
 *   AFPQ:  32-bit word[P] at 0: bits 0..15 = fp16 s+, bits 16..31 = fp16 s-.
 *   RaZeR: fp16 scale[P] at 0; 2-bit selectors from Z0 = round_up(2P, 256):
 *          selector of group f in byte Z0 + f/4, bits 2*(f%4)..2*(f%4)+1;
 *          the selector plane is round_up(ceil(P/4), 16) bytes long.
 *   INT8:  fp16 scale[N] at 0.
 *   FP16:  none (qnt_meta_bytes returns 0).
 * Every metadata length is rounded up to a multiple of 16 bytes (the GEMV
 * kernels stage whole 16-byte-aligned metadata ranges with bulk copies).
 */

/* Bytes of packed codes / metadata for a descriptor; 0 if it is invalid. */
size_t qnt_codes_bytes(const qnt_desc* desc);
size_t qnt_meta_bytes(const qnt_desc* desc);

/* Validate a descriptor: QNT_OK or the error code that the calls would return. */
int qnt_check_desc(const qnt_desc* desc);

/*
 * qnt_quantize -- RTN-quantize W into packed codes and metadata (the offline
 * step of the RTN page; data-free, no calibration).
 *   d_W        device, fp32 [N][K] row-major, read only.
 *   d_codes    device, qnt_codes_bytes(desc) bytes, written.
 *   d_meta     device, qnt_meta_bytes(desc) bytes, written (may be NULL for FP16).
 *   d_status   device int or NULL: QNT_ERR_NONFINITE / QNT_ERR_RANGE.
 * Bit-exact with the definitions above.  The call ends with an empty kernel on
 * the stream, so that a GEMV enqueued right after it (which requests its codes
 * and metadata before waiting for the preceding kernel, see qnt_gemv) sees them.
 */
int qnt_quantize(const qnt_desc* desc, const float* d_W, void* d_codes, void* d_meta,
                 int* d_status, void* stream);

/*
 * qnt_gemv -- batch-1 fused-dequant GEMV, y[n] = sum_k dq(n, k) * x[k]
 * (the decode-time GEMV of the RaZeR and RTN pages).
 *   d_codes, d_meta  device, packed as above (from qnt_quantize or the layout).
 *   d_x        device, [K] fp16 or bf16 (xdtype).
 *   d_y        device, [N] in the same type, written.
 *   d_status   device int or NULL: QNT_ERR_TIMEOUT if a staging wait expires.
 * Ordering (programmatic dependent launch): the GEMV kernels of qnt_gemv and
 * qnt_gemm start while the preceding kernel on the stream is still running and
 * request their codes and metadata at once; only the reads of x and the writes
 * of y wait for that kernel to complete.  So the kernel IMMEDIATELY preceding
 * the call on the stream must not write d_codes or d_meta.  qnt_quantize
 * complies (it ends with an empty kernel); after any other kernel that writes
 * the weights, enqueue another kernel or a copy in between, or synchronize.
 * Accuracy: |y - y_exact| <= 4e-3 * sum_k |dq(n,k) x[k]| per element.  Every
 * product is formed from exact fp16 operands and accumulated in fp32 (on the
 * CUDA cores exactly; on the tensor cores, which take batch 1 and larger
 * batches, within about 1e-4 of sum |products| as measured), with one final
 * rounding to the output type.  x is rescaled
 * internally by a power of two so fp16 arithmetic cannot overflow.
 */
int qnt_gemv(const qnt_desc* desc, const void* d_codes, const void* d_meta,
             const void* d_x, void* d_y, int xdtype, int* d_status, void* stream);

/*
 * qnt_gemm -- small-batch fused-dequant GEMM, Y[m][n] = sum_k dq(n, k) X[m][k]
 * for 1 <= M <= 128 activation rows.
 *   d_X        device, [M][K] fp16 or bf16, row-major.
 *   d_Y        device, [M][N] in the same type, written.
 * Same ordering rule (the immediately preceding kernel on the stream must not
 * write d_codes or d_meta) and accuracy statement as qnt_gemv.  Batches of 2 to
 * 8 rows of the 4-bit formats with group 128 and K a multiple of 1024 run on
 * the batch-1 kernel, the rows sharing its tensor-core MMAs, when their
 * activations fit in shared memory next to its weight ring; the other batches
 * of 3 to 128 rows of the 4-bit formats run on the tcgen05 tensor cores in one
 * pass over the weights.  d_status may also receive QNT_ERR_TIMEOUT on both.
 */
int qnt_gemm(const qnt_desc* desc, const void* d_codes, const void* d_meta,
             const void* d_X, void* d_Y, int M, int xdtype, int* d_status, void* stream);

/*
 * Sequences of batch-1 GEMVs in one launch: the linear layers of a decode step
 * (token generation with fused-dequant kernels, RTN and RaZeR pages' English
 * abstracts) run one after another on one activation vector each.  One
 * persistent kernel streams the weights of every step back to back; a step
 * with wait = k reads its x only after step i - k and every step before it
 * have written their y, so x may be (part of) one of those y.  (A decode layer:
 * o waits 1 for qkv, gate 1 for o, up 2 for o, down 1 for up.)
 */
#define QNT_SEQ_MAX_STEPS 256

typedef struct {
  qnt_desc desc;       /* 4-bit format, N, K, group: format and group equal in every step */
  const void* codes;   /* device, this step's packed codes */
  const void* meta;    /* device, its metadata */
  const void* x;       /* device, [K] activations (fp16 or bf16, as xdtype) */
  void* y;             /* device, [N] output, same type; written */
  int32_t wait;        /* k >= 1: read x after step i - k and every step before it
                          have written their y (x may be any of those y); 0: x is
                          not written by any earlier step of this call.  0 <= k <= i. */
  int32_t reserved;    /* 0 */
} qnt_seq_step;

/* Bytes of the workspace qnt_gemv_seq needs for nsteps steps (0 if nsteps is
 * out of range). */
size_t qnt_gemv_seq_work_bytes(int nsteps);

/*
 * qnt_gemv_seq -- y_i = W_i x_i for the steps i = 0 .. nsteps-1, in order.
 *   steps      HOST array of nsteps step descriptors (1 <= nsteps <=
 *              QNT_SEQ_MAX_STEPS); read during the call only.
 *   d_work     device, qnt_gemv_seq_work_bytes(nsteps) bytes, 16-byte aligned,
 *              owned by the caller: per-step completion counters.  The call
 *              clears it on the stream before the kernel; two calls that may
 *              run at the same time need two workspaces.
 *   d_status   device int or NULL: QNT_ERR_TIMEOUT if a wait expires (a step's
 *              dependency, a staging copy).
 * Step 0 starts after the preceding work on the stream has completed.  The y of
 * a step must not overlap any other step's y, x, codes or metadata except as
 * the x of a later step marked `wait`.  Accuracy as qnt_gemv.  The kernel keeps
 * one CTA on every SM for its whole duration (a cooperative launch);
 * QNT_ERR_CUDA if the GPU cannot host it.  QNT_ERR_ARG: nsteps out of range,
 * a null pointer, a format that is not 4-bit, formats / groups that differ
 * between steps, or wait outside 0..i; QNT_ERR_SHAPE / QNT_ERR_ALIGN as for
 * qnt_gemv, and QNT_ERR_SHAPE when a step's activations and staged metadata
 * do not fit in shared memory.
 */
int qnt_gemv_seq(const qnt_seq_step* steps, int nsteps, int xdtype, void* d_work, int* d_status, void* stream);

/*
 * qnt_gemv_seq_noalloc -- qnt_gemv_seq for callers that cannot allocate device
 * memory: for example a host framework whose device memory is entirely handed
 * out by its own pool, or a plug-in that is not allowed to call the CUDA
 * allocator, and so cannot provide d_work.  It computes exactly what
 * qnt_gemv_seq computes (same arguments, ordering, accuracy and errors) and
 * allocates nothing.  (No counterpart in the pages: an interface convenience.)
 *   Workspace: the per-step completion counters live in a small array that the
 *     library itself places in the memory of every GPU that loads it, for the
 *     life of the process ((QNT_SEQ_NOALLOC_MAX_STEPS + 1) * 4 bytes per GPU).
 *     Each call clears the part it uses on `stream` before its kernel; the
 *     array keeps the last call's contents afterwards.
 *   Limit: nsteps <= QNT_SEQ_NOALLOC_MAX_STEPS, else QNT_ERR_ARG.
 *   Every call shares the one array: two calls whose work overlaps on the GPU
 *     (other streams, other host threads) race and may hang until their waits
 *     expire (QNT_ERR_TIMEOUT); serialize them, or use qnt_gemv_seq with one
 *     workspace each.
 *   The first call on each device looks up the array's device address (a
 *     runtime query, no allocation); make that first call before capturing a
 *     stream into a CUDA graph.
 */
#define QNT_SEQ_NOALLOC_MAX_STEPS 256
int qnt_gemv_seq_noalloc(const qnt_seq_step* steps, int nsteps, int xdtype, int* d_status, void* stream);

/*
 * Selective precision (RTN page: raise the precision format of chosen layers
 * and modules).  A host-side table of ordered rules; qnt_table_lookup returns
 * the format and group of the first rule whose pattern matches the module name
 * ('*' matches any run of characters, '?' one character), else the default.
 * The table is a host object owned by the caller; not thread-safe for
 * concurrent modification.
 */
typedef struct qnt_table qnt_table;
qnt_table* qnt_table_create(int default_fmt, int default_group); /* NULL on bad args */
int qnt_table_set(qnt_table* t, const char* module_pattern, int fmt, int group);
int qnt_table_lookup(const qnt_table* t, const char* module_name, int* fmt, int* group);
int qnt_table_size(const qnt_table* t);
void qnt_table_destroy(qnt_table* t);

/* Static description of an error code. */
const char* qnt_strerror(int code);

/* After a call returned QNT_ERR_CUDA: the CUDA runtime's name and description
 * of the error, for the calling host thread ("" if none).  The text stays
 * valid until the thread's next failing call. */
const char* qnt_last_error(void);

/* Library version (QNT_VERSION of the build). */
int qnt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QNT_H_ */
