/*
 * q4_0.h -- C ABI of libq4_0_b200.so, the B200 (sm_100a) Q4_0 weight-only
 * dequantize-and-matmul library.
 *
 * The operation.  The pages run every decoder linear of the Voxtral 4B speech
 * models on 4-bit weights: "Q4_0 GGUF" weights through a custom fused
 * dequant+matmul shader (voxtral-mini-realtime-rs (Shannon-Prime fork)
 * README, "RTF Benchmark Results" and "Architecture Summary" (Q4 matmul
 * kernel per decoder layer); hakusoku.com story 5135, linear ops and
 * embeddings), with fused QKV and gate/up projections and batch-2 CFG
 * (voxtral-mini-realtime-rs README, "TTS (Text-to-Speech)", optimizations).
 * This library computes
 *
 *     Y[M,N] = X[M,K] * dequant(W)^T
 *
 * where
 *   W  is N rows of K weights in Q4_0 blocks: each run of 32 weights of a row
 *      is 18 bytes = fp16 scale d (little-endian) + 16 bytes qs, byte j of qs
 *      holding code q[j] (low nibble) and q[j+16] (high nibble); a weight is
 *      w = (q - 8) * d; blocks of a row are contiguous and rows follow each
 *      other with no padding (row size K/32*18 bytes);
 *   X  is bf16, row-major [M,K] (row stride K elements);
 *   Y  is fp32, row-major [M,N] (row stride N elements), overwritten.
 * Accumulation is fp32.  Results agree with the exact (float64) product to
 * |Y - Y_exact| <= 1e-3 * sum_k |X[m,k] * w[n,k]| + 1e-6 per element; pack and
 * dequant are bit-exact.
 *
 * Conventions for every entry point:
 *   * all data pointers are DEVICE pointers owned by the caller; the library
 *     never frees, keeps or allocates them, and allocates nothing per call;
 *   * `stream` is a cudaStream_t (NULL = the legacy default stream); every
 *     call is asynchronous on it and returns without a host synchronisation;
 *   * arguments are checked on the host before anything is launched; on a
 *     failed check nothing is launched and a status != Q4_OK is returned;
 *   * sizes are element counts; a size of 0 is valid (see each call);
 *   * the calling thread's current CUDA device must be an sm_100 GPU (compute
 *     capability 10.0), else Q4_ERR_UNSUPPORTED_DEVICE.
 * Asynchronous faults surface on the stream as for any CUDA kernel.  Kernels
 * that wait on on-chip barriers bound every wait; a wait that runs out sets a
 * device-side error word (q4_0_device_error) and the kernel returns early.
 */
#ifndef Q4_0_B200_H
#define Q4_0_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define Q4_0_API __attribute__((visibility("default")))
#else
#define Q4_0_API
#endif

/* Same type as cudaStream_t, declared here so that this header needs no CUDA
 * header. */
typedef struct CUstream_st *q4_0_stream_t;

enum {
    Q4_OK = 0,
    Q4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, K % 32 != 0, too large */
    Q4_ERR_MISALIGNED = 2,         /* a pointer is not 16-byte aligned */
    Q4_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not compute capability 10.0 */
    Q4_ERR_CUDA = 4,               /* a CUDA runtime call failed; see q4_0_last_cuda_error */
    Q4_ERR_TOO_LARGE = 5           /* the problem needs more scratch than Q4_0_STATIC_WS_BYTES */
};

/* Device error bits reported by q4_0_device_error. */
enum {
    Q4_DEVERR_WAIT_TIMEOUT = 1u,   /* a bounded on-chip wait gave up; the output is incomplete */
    Q4_DEVERR_BAD_INDEX = 2u,      /* q4_0_gather met an id outside [0, V) (its row was zeroed) */
    Q4_DEVERR_FP16_RANGE = 4u,     /* a fast GEMM path met an operand too large for its fp16
                                      arithmetic: a finite X with |x| > 65504, or a scale with
                                      8188 < |d| < inf; its output may hold +-inf (q4_0_force_path(4)
                                      computes such inputs exactly) */
    Q4_DEVERR_DEBUG_CHECK = 8u     /* only in a library built with Q4_DEBUG defined: an index check
                                      found a shared- or tensor-memory index outside its buffer; the
                                      access was skipped and the kernel stopped early */
};

/* Largest N, K and M accepted (each dimension below 2^31). */
#define Q4_0_MAX_DIM 2147483647LL

/* Human-readable name of a status code; never NULL. */
Q4_0_API const char *q4_0_status_string(int status);

/* The cudaError_t of the last call that returned Q4_ERR_CUDA on this thread
 * (0 if none). */
Q4_0_API int q4_0_last_cuda_error(void);

/* Bytes of a Q4_0 matrix of N rows by K weights: N * (K/32) * 18.  Returns -1
 * if N < 0, K < 0 or K % 32 != 0. */
Q4_0_API int64_t q4_0_bytes(int64_t N, int64_t K);

/* Pack 4-bit codes and fp16 scales into Q4_0 blocks (bit-exact).
 *   codes  [N,K] uint8, row-major; only the low nibble of each byte is used;
 *   scales [N,K/32] uint16 fp16 bit patterns, row-major (scale of block
 *          k/32 of row n at scales[n*(K/32) + k/32]);
 *   W      output, q4_0_bytes(N,K) bytes, layout as above.
 * codes, scales and W must be 16-byte aligned.  K % 32 == 0.  N == 0 or
 * K == 0 writes nothing.  The GGUF Q4_0 packing is the reading taken of the
 * pages' "Q4_0 GGUF" (voxtral-mini-realtime-rs README, "RTF Benchmark
 * Results"); codes are given, not derived from float weights. */
Q4_0_API int q4_0_pack(const uint8_t *codes, const uint16_t *scales, void *W,
              int64_t N, int64_t K, q4_0_stream_t stream);

/* Dequantize Q4_0 blocks to fp32: out[n,k] = (q - 8) * d, exact (bit-exact
 * against any correct implementation).  W as in q4_0_pack; out [N,K] fp32
 * row-major.  W and out 16-byte aligned.  N == 0 or K == 0 writes nothing.
 * This is the dequantization half of the fused shader (hakusoku.com story
 * 5135, linear ops and embeddings) on its own, for tests and utilities. */
Q4_0_API int q4_0_dequant(const void *W, float *out, int64_t N, int64_t K,
                 q4_0_stream_t stream);

/* Y[M,N] = X[M,K] * dequant(W)^T with fp32 accumulation, W never written out
 * dequantized (the fused dequant+matmul of hakusoku.com story 5135, linear
 * ops and embeddings; one Q4 matmul per decoder linear as in
 * voxtral-mini-realtime-rs README, "Architecture Summary").
 *   W  Q4_0 [N, K/32 blocks], X bf16 bit patterns [M,K], Y fp32 [M,N].
 *   W, X, Y must be 16-byte aligned; K % 32 == 0; X and Y must not overlap W
 *   or each other.
 *   M == 0 or N == 0: nothing is done.  K == 0: Y is filled with zeros.
 * Path: M <= 32 runs the memory-bound decode kernel (weights dequantized in
 * registers, products on the warp-level tensor cores); M > 32 runs the
 * tcgen05 tensor-core kernel (weight tiles dequantized into tensor memory,
 * fp32 accumulators in tensor memory).  Both feed the tensor cores fp16
 * operands: each weight (q - 8) * d is rounded once to fp16 (relative error
 * <= 2^-11) and X is converted to fp16: exactly for 2^-17 <= |x| <= 65504,
 * with an absolute error below 2^-25 for smaller |x|.  An operand too large
 * for fp16 (a finite |x| > 65504, a scale 8188 < |d| < inf) is detected on
 * the GPU and sets Q4_DEVERR_FP16_RANGE in q4_0_device_error: the output may
 * then hold +-inf.  q4_0_force_path(4) selects an exact-arithmetic decode
 * kernel ((q - 8) exact in bf16, X used as given) without that restriction. */
Q4_0_API int q4_0_gemm(const void *W, const uint16_t *X, float *Y,
              int64_t M, int64_t N, int64_t K, q4_0_stream_t stream);

/* Bytes of device workspace q4_0_gemm_ws can use for an (M, N, K) problem:
 * M*K*2 rounded up to 256 when M > 32 (an fp16 copy of X for the
 * tensor-core path), 0 when M <= 32.  -1 for invalid sizes. */
Q4_0_API int64_t q4_0_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/* q4_0_gemm with a caller-provided device workspace (16-byte aligned, owned
 * by the caller, contents overwritten).  With workspace_bytes >=
 * q4_0_gemm_workspace_size(M, N, K), the tensor-core path (M > 32) first
 * converts X to fp16 once in the workspace (one extra read and write of X)
 * instead of converting every X tile in every CTA that loads it; with a
 * smaller or NULL workspace it behaves exactly as q4_0_gemm.  The library
 * never writes past workspace_bytes: the conversion runs only when the
 * workspace holds all M*K*2 bytes (rounded up to 256) that it writes.  Same results,
 * bit for bit, either way.  Calls that share one workspace and overlap on
 * the GPU race.  The pages have no counterpart: this is the B200 path's own
 * trade of one pass over X against per-tile conversion work. */
Q4_0_API int q4_0_gemm_ws(const void *W, const uint16_t *X, float *Y,
                          int64_t M, int64_t N, int64_t K, void *workspace,
                          int64_t workspace_bytes, q4_0_stream_t stream);

/* The two phases of q4_0_gemm_ws's tensor-core path as separate calls, so
 * that a caller can convert the X of the next GEMM while the current one runs
 * (on another stream: the conversion reads and writes HBM while the GEMM
 * keeps the tensor cores busy), or convert an X once for several GEMMs that
 * share it.  No counterpart on the pages: the same trade as q4_0_gemm_ws.
 *
 * q4_0_prepared_x_bytes: bytes of the prepared copy of an [M, K] X:
 * M*K*2 rounded up to 256; -1 for a negative or too large M or K, or K not a
 * multiple of 256.
 *
 * q4_0_prepare_x: writes bf16 X [M, K] (device, 16-byte aligned, row-major)
 * into `xh` (device, 16-byte aligned, owned by the caller, at least
 * q4_0_prepared_x_bytes(M, K) bytes, else Q4_ERR_INVALID_ARG) as fp16 in the
 * order the tensor-core kernel reads (within every 4 consecutive k, positions
 * 1 and 2 swapped).  A finite |x| > 65504 sets Q4_DEVERR_FP16_RANGE.
 *
 * q4_0_gemm_prepared: Y[M,N] = X * dequant(W)^T on the tensor-core kernel
 * whatever M is, reading X from `xh` as written by q4_0_prepare_x for the
 * same M and K (device pointers, 16-byte aligned; K a positive multiple of
 * 256, else Q4_ERR_INVALID_ARG).  For M > 32 the result is that of
 * q4_0_gemm_ws (and so q4_0_gemm) bit for bit.  The order between the two
 * calls is the caller's: the same stream, or an event. */
Q4_0_API int64_t q4_0_prepared_x_bytes(int64_t M, int64_t K);
Q4_0_API int q4_0_prepare_x(const uint16_t *X, int64_t M, int64_t K, void *xh, int64_t xh_bytes,
                            q4_0_stream_t stream);
Q4_0_API int q4_0_gemm_prepared(const void *W, const void *xh, float *Y, int64_t M, int64_t N, int64_t K,
                                q4_0_stream_t stream);

/* Size of the library's fixed device scratch array used by
 * q4_0_gemm_static_ws: 64 MiB on each device (an fp16 copy of X up to
 * M*K = 32 Mi elements, e.g. M = 4096 rows at K = 8192). */
#define Q4_0_STATIC_WS_BYTES (64LL << 20)

/* q4_0_gemm_ws with the library's own fixed scratch array as the workspace:
 * it never allocates device memory (no cudaMalloc, no allocating library
 * routine).  For callers that may not allocate device memory when they
 * multiply: a real-time audio thread that must not block in an allocator, a
 * process that budgets device memory once at start-up, code that runs where
 * no device allocator is reachable.
 *   * Host memory: the library's small host-side caches (per-thread problem
 *     lists, the cache of TMA descriptors, guarded by a mutex) grow on a
 *     thread's first call and on the first call with each new W or X pointer
 *     or shape.  A caller that must not touch the host allocator either
 *     makes one call with each of its buffers and shapes first, off the
 *     real-time thread, or takes the library's host-side growth into account.
 *   * The array (Q4_0_STATIC_WS_BYTES, 256-byte aligned) is a __device__
 *     variable of the library, one copy per device.  A problem whose
 *     workspace size (q4_0_gemm_workspace_size) exceeds it is rejected with
 *     Q4_ERR_TOO_LARGE and nothing is launched; M <= 32 needs none (a
 *     tensor-core run forced for M <= 32 uses the array only when its fp16
 *     copy of X fits, and otherwise converts X tile by tile).
 *   * Nothing in the array has to start at zero: each call writes every byte
 *     it reads before reading it, on `stream`.
 *   * Calls whose kernels can overlap on one device (different streams or
 *     host threads without ordering between them) share the array and race;
 *     calls on one stream, or otherwise ordered, are safe.
 *   * The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current, which may load the
 *     library module holding it); make that first call before any stream
 *     capture begins.  Every call needs a current sm_100 device, even one
 *     with nothing to compute.
 * Results are those of q4_0_gemm_ws with a large enough workspace (the same
 * as q4_0_gemm, bit for bit).  The pages have no counterpart: this is a
 * deployment convenience of this library. */
Q4_0_API int q4_0_gemm_static_ws(const void *W, const uint16_t *X, float *Y,
                                 int64_t M, int64_t N, int64_t K, q4_0_stream_t stream);

/* Fused epilogues (q4_0_gemm_grouped_ex). */
#define Q4_0_EPI_NONE 0      /* Y = X * dequant(W)^T */
#define Q4_0_EPI_RESIDUAL 1  /* Y = X * dequant(W)^T + R (R [M,N] fp32; R == Y allowed) */
#define Q4_0_EPI_SWIGLU 2    /* Y[M, N/2] = silu(gate) * up of a row-interleaved gate/up W */

/* A grouped problem with a fused epilogue.  W, X, M, N, K as in
 * q4_0_problem.  R: the residual for Q4_0_EPI_RESIDUAL (device, 16-byte
 * aligned, [M,N] fp32), ignored otherwise.  For Q4_0_EPI_SWIGLU, W holds 2F
 * rows (N = 2F, F % 64 == 0) in the order q4_0_interleave_gate_up writes
 * and Y is [M, F]. */
typedef struct q4_0_problem_ex {
    const void *W;
    const uint16_t *X;
    float *Y;
    int64_t M, N, K;
    const float *R;
    int32_t epilogue;
} q4_0_problem_ex;

/* q4_0_gemm_grouped with the step on either side of a decoder layer's
 * linears fused into the store of Y, so that no intermediate makes a round
 * trip through HBM: the residual add after the O and down projections, and
 * the SwiGLU activation silu(g) * u (silu(g) = g / (1 + exp(-g)), fp32)
 * between the fused gate/up projection (voxtral-mini-realtime-rs README, TTS
 * section, optimizations) and the down projection.  Problems with M <= 32
 * run on the decode path (all of them in one launch); each problem with
 * M > 32 runs on the tensor-core kernel, whose epilogue warps apply its
 * epilogue as they drain the accumulator (X converted to fp16 tile by tile,
 * no workspace).  Every problem needs M >= 1, K a positive multiple of 256
 * and 16-byte aligned W, X, Y, R, else Q4_ERR_INVALID_ARG and nothing is
 * launched.  Tolerance: the GEMM bound of each input of the epilogue, carried
 * through it (silu' <= 1.1), plus fp32 rounding of the epilogue. */
Q4_0_API int q4_0_gemm_grouped_ex(const q4_0_problem_ex *problems, int count, q4_0_stream_t stream);

/* Row-interleaved gate/up weight for Q4_0_EPI_SWIGLU: W_gu rows 128i .. 128i+63
 * = W_gate rows 64i .. 64i+63 and rows 128i+64 .. 128i+127 = W_up rows
 * 64i .. 64i+63, for i < F/64.  W_gate, W_up: F rows each; W_gu: 2F rows; all
 * Q4_0 device buffers, 16-byte aligned, not overlapping; F % 64 == 0 and
 * K % 256 == 0. */
Q4_0_API int q4_0_interleave_gate_up(const void *W_gate, const void *W_up, void *W_gu,
                                     int64_t F, int64_t K, q4_0_stream_t stream);

/* Self-test of the failure detection (no counterpart on the pages): one
 * CTA waits on an on-chip barrier that nothing arrives on, bounded by
 * limit_us (1 .. 1000000); the wait gives up, ORs Q4_DEVERR_WAIT_TIMEOUT into
 * q4_0_device_error and the kernel returns, leaving the context usable.  It
 * lets a test show that a bounded wait ends and reports, without any fault.
 * Asynchronous on `stream` like every call. */
Q4_0_API int q4_0_selftest_wait_timeout(uint32_t limit_us, q4_0_stream_t stream);

/* A measurement instrument (no counterpart on the pages): read the Q4_0
 * matrix W (N rows, K weights each) once from device memory with the same
 * weight stream the decode kernels use -- TMA boxes of 128 rows x 144 bytes
 * (256 k) into a ring of shared-memory slots, one persistent CTA per SM,
 * each CTA walking along K of one 128-row item and then the next -- and do
 * nothing with the bytes but XOR their 32-bit words into *checksum (a device
 * word the caller initialises; rows past N read as zero).  The bandwidth this
 * reaches is the ceiling of the decode kernels' access pattern: what they
 * would stream if their arithmetic were free.  W 16-byte aligned, checksum
 * 4-byte aligned, K % 256 == 0; N == 0 or K == 0 is a no-op. */
Q4_0_API int q4_0_stream_read(const void *W, int64_t N, int64_t K, uint32_t *checksum, q4_0_stream_t stream);

/* Row gather (a Q4 embedding lookup): out[t, :] = dequant(W)[ids[t], :] for
 * t < T, W a Q4_0 matrix of V rows by D weights, out float32 [T, D] row-major
 * (exact: each (q - 8) * d is representable in float32).  The pages keep the
 * 131072 x 3072 token embeddings of the Voxtral models in Q4 and dequantize
 * the looked-up rows on the host (hakusoku.com story 5135, linear ops and
 * embeddings; voxtral-mini-realtime-rs README, "WASM Constraints Solved",
 * item 3); this is that step on the GPU.  ids: int32 device array of T
 * entries (4-byte aligned); W and out 16-byte aligned; D % 32 == 0.  An id
 * outside [0, V) -- which the host cannot see without a synchronisation --
 * gives a row of zeros and sets Q4_DEVERR_BAD_INDEX in q4_0_device_error.
 * T == 0 or D == 0 is a no-op; V must be >= 1 otherwise. */
Q4_0_API int q4_0_gather(const void *W, const int32_t *ids, float *out,
                         int64_t T, int64_t V, int64_t D, q4_0_stream_t stream);

/* Quantize float32 weights X[N, K] (row-major, finite) to Q4_0 blocks W
 * (N * K/32 * 18 bytes) by the GGUF Q4_0 rule that the pages apply offline
 * (their quantize_tts_gguf.py, voxtral-mini-realtime-rs README, TTS section;
 * the rule itself is not on the pages): per block of 32, m = the value of
 * largest magnitude (the first on ties, +0 for an all-zero block),
 * d = m / -8, id = 1/d (0 when d == 0), q = min(15, trunc(x * id + 8.5)) in
 * float32 with the product rounded before the sum; the block stores fp16(d)
 * rounded to nearest even.  Deterministic and bit-exact.  X and W 16-byte
 * aligned, K % 32 == 0; N == 0 or K == 0 is a no-op. */
Q4_0_API int q4_0_quantize(const float *X, void *W, int64_t N, int64_t K, q4_0_stream_t stream);

/* One problem of a grouped launch: Y = X * dequant(W)^T, all device
 * pointers, same rules as q4_0_gemm. */
typedef struct q4_0_problem {
    const void *W;
    const uint16_t *X;
    float *Y;
    int64_t M, N, K;
} q4_0_problem;

/* Largest `count` accepted by q4_0_gemm_grouped. */
#define Q4_0_MAX_GROUP 256

/* Run `count` independent problems in as few launches as possible (one
 * persistent launch for all problems with M <= 32), so that a decoder
 * layer's QKV, O, gate/up and down projections -- or all layers of a decode
 * step -- stream their weights in one pass without a launch and a tail per
 * linear (the fused QKV and gate/up projections of voxtral-mini-realtime-rs
 * README, "TTS (Text-to-Speech)", optimizations, generalised to whole
 * layers).  `problems` is a HOST array read during the call (it may be
 * reused as soon as the call returns).  0 <= count <= Q4_0_MAX_GROUP.  All
 * problems are checked before anything is launched. */
Q4_0_API int q4_0_gemm_grouped(const q4_0_problem *problems, int count,
                      q4_0_stream_t stream);

/* Read (and, if clear != 0, reset) the device error word of the current
 * device: an OR of Q4_DEVERR_* bits set by kernels since the last reset.
 * Synchronises the device.  The pages have no counterpart; this is the
 * library's failure-detection hook. */
Q4_0_API int q4_0_device_error(uint32_t *flags, int clear);

/* Testing knob, process-wide: force the kernel family used by q4_0_gemm and
 * q4_0_gemm_grouped.  0 = automatic (default), 1 = portable kernel (any
 * shape), 2 = decode kernel (M <= 32 only), 3 = tensor-core kernel, 4 = the
 * exact-arithmetic decode kernel ((q - 8) exact in bf16, d applied in fp32;
 * M <= 32), 5 = the tcgen05 decode kernel (weights in tensor memory; M <= 32),
 * 6 = the M <= 8 decode kernel with 512-k ring slots (automatic for M <= 8;
 * path 2 sends M <= 8 to the kernel with 256-k stages instead).
 * A forced family that cannot run a given shape falls back to automatic.  The
 * pages have no counterpart. */
Q4_0_API int q4_0_force_path(int path);

#ifdef __cplusplus
}
#endif

#endif /* Q4_0_B200_H */
