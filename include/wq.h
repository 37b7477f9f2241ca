/*
 * wq.h — C ABI of libwq.so: weight-only quantized decode linear layer
 * y = x·Wᵀ for B200 (sm_100a), with W dequantized on the fly.
 *
 * Shapes: x is [M, K] row-major, W is logically [N, K], y is [M, N] row-major.
 * M is the decode batch (the GEMV family serves M = 1..8; M >= 9 runs the
 * batched family: for B200_V1 int4 the tcgen05 dequant-then-MMA kernel from
 * M = 25, and from M = 9 when its 128-row tiles alone fill the GPU, else a
 * warp-MMA GEMM over the band stream; for the canonical formats the tcgen05
 * kernel where it applies, else the GEMV in chunks of 8 rows of x), N the
 * output features, K the input features.  Every
 * floating-point result is accumulated in fp32.
 *
 * Conventions for every entry point below:
 *  - Pointers named *_host are host pointers; every other pointer is a CUDA
 *    device pointer owned by the caller.  The library never frees, keeps or
 *    allocates memory on these paths, and it has no CPU fallback.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Launch entry points are asynchronous on that stream; they return after
 *    enqueueing.  Argument errors are reported before anything is enqueued.
 *  - Return value: WQ_OK (0) or a negative WQ_ERR_* code.  wq_last_error()
 *    then holds a one-line message (per calling thread).
 *  - wq_last_kernel() names the kernel variant the last successful launch on
 *    the calling thread used (a liveness label such as
 *    "int4.gemv.v1s.m1.c1"), so a test can assert which path ran.
 *  - The decode GEMV kernels are launched with programmatic dependent launch:
 *    a call may start while the previous kernel in the stream is still
 *    running.  Until that kernel has completed, a call only prefetches the
 *    head of its weight stream into L2 (L2 is the point of coherence, so this
 *    can never return data older than a write of that kernel); it copies
 *    weights into shared memory or registers, reads x and writes y only
 *    after waiting for the previous kernel to complete.  The previous kernel
 *    may therefore write this call's weights (a repack, an upload kernel)
 *    with no synchronization in between.  A following kernel that itself
 *    uses programmatic dependent launch must wait (griddepcontrol.wait)
 *    before reading y, as usual.
 *  - The tensor-core family (M >= 9) forms each weight in fp16 (q4_K, int4)
 *    before the MMA, rounded once (relative error <= 2^-11 per weight).  A
 *    weight row whose bound could pass the fp16 range (15·max|s| for int4,
 *    max(|d|·945 + |dmin|·63) over the super-blocks for q4_K, above 65504)
 *    is formed as w·2^-e with the least such e, and its fp32 result is
 *    multiplied by 2^e: no finite weight becomes infinite.  In such a row a
 *    weight that falls below the fp16 normal range after the scaling keeps
 *    an absolute error of at most 2^(e-25).
 *  - The first call on a device configures kernel attributes and looks up the
 *    driver's tensor-map encoder; make it before capturing a CUDA graph.
 *  - Environment variables read at each call, for tests and tuning only:
 *    WQ_FORCE_KERNEL (tc | cc | simple | tc5 | v1s | v1r | v1k | v1tc | v1w | mx | mmq) pins a kernel
 *    family (a call that family cannot run returns WQ_ERR_UNSUPPORTED; there
 *    is no silent substitute), WQ_PDL=0 disables programmatic dependent
 *    launch, and WQ_V1_*, WQ_V1R_*, WQ_V1K_*, WQ_V1W_*, WQ_V1TC_*, WQ_TC_*,
 *    WQ_TC5_S, WQ_TC5_TA and WQ_MMQ_* override launch geometry (WQ_V1TC_TA=0 and
 *    WQ_TC5_TA=0 keep the tcgen05 kernels' fp16 A rows in shared memory
 *    instead of tensor memory; same results within the tolerance, slower).
 *
 * Weight formats (canonical byte layouts, layout version WQ_LAYOUT_CANONICAL):
 *  - int4 MatMulNBits-style blocks (onnx-genai PR #1000, "What it does": int4
 *    blockwise weights with fp16 scales and zero-points).  w_packed is
 *    [N][K/2] bytes, two 4-bit codes per byte, low nibble = even k.  A row
 *    has nb = ceil(K/block_size) blocks along K; when K is not a multiple of
 *    block_size the last one is shorter (K - (nb-1)·block_size codes, no
 *    padding in the code array).  scales is [N][nb] fp16.  zeros is
 *    [N][ceil(nb/2)] bytes, two uint4 zero-points per byte, low nibble = even
 *    block; NULL means z = 8 for every block.  w = (q - z)·s.
 *  - q4_K super-blocks (minfer doc 62 "r59 — q4_K W_dsc plane", §3.2): row n
 *    holds K/256 blocks of 144 bytes: fp16 d (bytes 0-1), fp16 dmin (2-3),
 *    12 bytes of packed 6-bit scales and mins (4-15), 128 bytes of 4-bit
 *    codes (16-143) in four runs of 32 bytes, run p holding chunk 2p in its
 *    low nibbles and chunk 2p+1 in its high nibbles.  For the 32-element
 *    chunk c of a block, w = d·sc_c·q - dmin·m_c (§2.1).
 *  - W_dsc plane (same page, §2.2): for global chunk c = 8·block + j and row
 *    n, the float2 (d·sc_j, -(dmin·m_j)), each one fp32 multiply, stored
 *    chunk-major at byte offset (c·N + n)·8: (K/32)·N float2 = N·K/4 bytes.
 *  - bf16: W [N][K] row-major, x [M][K] row-major, any K >= 1 and any 2-byte
 *    aligned base (AstrAI commit log, astrai/extension/backend: the bf16 GEMV
 *    accepts any K and any storage offset).
 *
 * Alignment: the int4 and q4_K entry points need 16-byte aligned device
 * pointers (cudaMalloc and PyTorch allocations are); otherwise they return
 * WQ_ERR_ALIGN.  The bf16 entry points accept any 2-byte aligned pointers.
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define WQ_OK 0
#define WQ_ERR_ARG (-1)         /* bad pointer, dimension, block size or layout value */
#define WQ_ERR_ALIGN (-2)       /* a device pointer is not 16-byte aligned (int4, q4_K) */
#define WQ_ERR_LAYOUT (-3)      /* weights were packed for another layout version */
#define WQ_ERR_CUDA (-4)        /* a CUDA runtime call or launch failed; see wq_last_error() */
#define WQ_ERR_DEVICE (-5)      /* the current device is not sm_100 */
#define WQ_ERR_TIMEOUT (-6)     /* a bounded device-side wait expired (see wq_device_status) */
#define WQ_ERR_UNSUPPORTED (-7) /* valid arguments this library version has no kernel for */

/* Weight layout versions. */
#define WQ_LAYOUT_CANONICAL 0
/* B200_V1 (int4): the codes, scales and zero-points of 16-row bands stored as
 * one contiguous stream per band, read front to back.  Rows are grouped in
 * bands of 16 (the last band padded with zero codes, scale 0, zero-point 8).
 * A band is K/128 consecutive tiles of WQ_INT4_V1_TILE_BYTES(block_size)
 * bytes; tile s covers k = 128s .. 128s+127 of the band's 16 rows:
 *   bytes [0, 1024): codes in warp-MMA fragment order: offset h·512 + lane·16
 *     + 4·(2·(gi & 1) + r8) holds the 32-bit code word of band row
 *     (lane / 4) + 8·r8 for k = 128s + 32·gi + 8·(lane % 4) + e, e = 0..7
 *     (gi = 2h + (0|1)), code e in nibble position (e >> 1) | ((e & 1) << 2);
 *   then bpt = max(1, 128 / block_size) scale rows [bpt][16] fp16 (for
 *     block 256 each tile repeats its block's scales);
 *   then zero-points [bpt][8] bytes (row 2i low nibble, row 2i+1 high);
 *   padded to a multiple of 16 bytes.
 * Needs K % 128 == 0 and block_size >= 32.  Built on the device by
 * wq_repack_int4 (onnx-genai PR #1000, "Roadmap recommendation": an offline
 * interleaving repack behind a versioned layout flag).  With this layout the
 * GEMV ignores its scales and zeros arguments (they may be NULL). */
#define WQ_INT4_V1_TILE_BYTES(bs) \
  ((1024 + ((bs) >= 128 ? 1 : 128 / (bs)) * 40 + 15) / 16 * 16)
#define WQ_LAYOUT_B200_V1 1
/* B200_V1 (q4_K): the same band idea for q4_K super-blocks.  Rows are grouped
 * in bands of 16 (the last band padded with zero codes and zero d, dmin and
 * scales); a band is K/256 consecutive tiles of WQ_Q4K_V1_TILE_BYTES bytes,
 * tile s holding super-block s of the band's 16 rows (exactly the 16 × 144
 * canonical bytes, reordered; minfer doc 62 "r59 — q4_K W_dsc plane", §3.2
 * for the canonical fields):
 *   bytes [0, 2048): codes in warp-MMA fragment order: offset h·512 + lane·16
 *     + 4·(2·(gi & 1) + r8) holds the 32-bit code word of band row
 *     (lane / 4) + 8·r8 for k = 256s + 32·gi + 8·(lane % 4) + e, e = 0..7
 *     (gi = 2h + (0|1) = the 32-element chunk, h = 0..3), code e in nibble
 *     position (e >> 1) | ((e & 1) << 2);
 *   bytes [2048, 2112): the rows' (d, dmin) fp16 pairs, 4 bytes per row;
 *   bytes [2112, 2304): 24-bit little-endian entries, entry (pair p, row r) at
 *     2112 + 3·(16p + r) = sc_{2p} | sc_{2p+1} << 6 | m_{2p} << 12 |
 *     m_{2p+1} << 18 (the 6-bit scales and mins of chunks 2p, 2p+1, §2.1).
 * Built on the device by wq_repack_q4k. */
#define WQ_Q4K_V1_TILE_BYTES 2304

/* ---------------------------------------------------------------------------
 * GEMV / GEMM entry points.  All device pointers; y is written, never read.
 * ------------------------------------------------------------------------- */

/* y[M,N] fp16 = x[M,K] fp16 · dequant(int4)ᵀ.
 * block_size: a power of two in [16, 256]; K % 16 == 0 (K need not be a
 * multiple of block_size: the last block of a row is then shorter).
 * zeros_u4 may be NULL (z = 8).  layout: WQ_LAYOUT_CANONICAL, or
 * WQ_LAYOUT_B200_V1 for weights rewritten by wq_repack_int4 (then w_packed is
 * the repacked buffer and scales_f16 / zeros_u4 are ignored).
 * M >= 1, N >= 1, K >= 1.  Errors: WQ_ERR_ARG, WQ_ERR_ALIGN, WQ_ERR_LAYOUT,
 * WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int gemv_int4_blockwise(const void* x_f16, const void* w_packed, const void* scales_f16,
                        const void* zeros_u4, void* y_f16, int M, int N, int K,
                        int block_size, int layout, void* stream);

/* Fused gate / up projection of a SwiGLU feed-forward block:
 *   y[M,N] fp16 = silu(x·W_gateᵀ) ⊙ (x·W_upᵀ),  silu(a) = a·σ(a) = a / (1 + e^-a),
 * both projections accumulated in fp32 from the same resident activations and
 * combined in fp32 before the one rounding to fp16 (the fused "swiglu" launch
 * of minfer doc 62 "r59 — q4_K W_dsc plane", §3.3; the page names the launch,
 * the formula is the SwiGLU definition).  w_gate_up is the fused B200_V1
 * stream of wq_repack_int4_gate_up: in every 16-row band, the tiles alternate
 * gate tile s, up tile s (each a B200_V1 int4 tile).  block_size 128 or 256,
 * K % 128 == 0, layout WQ_LAYOUT_B200_V1; up to 8 rows of x per launch whose
 * activations fit in 120 KB (more rows run in chunks).  Errors: WQ_ERR_ARG,
 * WQ_ERR_ALIGN, WQ_ERR_LAYOUT, WQ_ERR_UNSUPPORTED (K too large), WQ_ERR_DEVICE,
 * WQ_ERR_CUDA. */
int gemv_int4_swiglu(const void* x_f16, const void* w_gate_up, void* y_f16, int M, int N, int K,
                     int block_size, int layout, void* stream);

/* y[M,N] fp16 = x[M,K] fp16 · dequant(q4_K)ᵀ, scales decoded in-kernel from
 * the packed 6-bit fields.  K % 256 == 0.  w_q4k is N·(K/256)·144 bytes. */
int gemv_q4k(const void* x_f16, const void* w_q4k, void* y_f16, int M, int N, int K,
             int layout, void* stream);

/* gemv_q4k for the B200_V1 q4_K stream, for callers that must not allocate
 * device memory.  No counterpart on the pages: it exists because the ordinary
 * call sets up a small split-band workspace with cudaMalloc the first time it
 * runs on a stream, and some callers cannot allow that: programs that own all
 * device memory through their own pool or a fixed budget, and programs that
 * must not let a library call block or synchronize the device the way
 * cudaMalloc can.  This call instead uses one fixed array in the library's
 * own device memory (about 272 KB, reserved on every GPU that loads the
 * library and held until the process exits); it never calls cudaMalloc or
 * cudaFree.  Its first call on a device looks up the array's device address;
 * make that first call before any stream capture.  Limits: layout must be
 * WQ_LAYOUT_B200_V1, N <= 65536 (larger N returns WQ_ERR_ARG); the other
 * arguments are those of gemv_q4k.  The array keeps the last call's contents
 * and each call clears the part that must start at zero, so calls that
 * overlap on the GPU (for example on two streams at once) race: run them one
 * after another.  Errors: WQ_ERR_ARG, WQ_ERR_ALIGN, WQ_ERR_LAYOUT,
 * WQ_ERR_UNSUPPORTED, WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int gemv_q4k_noalloc(const void* x_f16, const void* w_q4k, void* y_f16, int M, int N, int K, int layout,
                     void* stream);

/* As gemv_q4k, but the per-chunk coefficients come from the W_dsc plane w_dsc
 * ((K/32)·N float2, chunk-major, N·K/4 bytes; build it with wq_build_q4k_dsc or
 * wq_build_q4k_dsc_device).  Only the code bytes of w_q4k are read. */
int gemv_q4k_dsc(const void* x_f16, const void* w_q4k, const void* w_dsc, void* y_f16,
                 int M, int N, int K, int layout, void* stream);

/* y[M,N] bf16 = x[M,K] bf16 · W[N,K]ᵀ bf16.  Any K >= 1; x, w, y only need
 * 2-byte alignment (rows of W and x are contiguous with stride K). */
int gemv_bf16(const void* x_bf16, const void* w_bf16, void* y_bf16, int M, int N, int K,
              void* stream);

/* y[M,N] fp16 = x[M,K] fp16 · W[N,K]ᵀ, W mxfp4 blockwise (onnx-genai PR #1000,
 * CPU criterion bench block: the mxfp4 block-quantized matmul rows; the page
 * does not print the format, the reading is the OCP microscaling FP4
 * definition): blocks of 32 elements along K share one E8M0 scale byte E,
 * value 2^(E - 127) (E = 255 is NaN), and every element is a 4-bit E2M1 code
 * (bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa; values 0, 0.5,
 * 1, 1.5, 2, 3, 4, 6 and their negatives).
 *   w_packed     codes [N][K/2] bytes, low nibble = even k (16-byte aligned)
 *   scales_e8m0  [N][K/32] bytes (any alignment)
 * K % 32 == 0 (else WQ_ERR_ARG).  fp32 accumulation; each block's scale is
 * applied in fp32.  Batches past 8 rows run in chunks of 8 (W read once per
 * chunk).  WQ_FORCE_KERNEL other than "mx" returns WQ_ERR_UNSUPPORTED. */
int gemv_mxfp4(const void* x_f16, const void* w_packed, const void* scales_e8m0, void* y_f16, int M, int N, int K,
               void* stream);

/* ---------------------------------------------------------------------------
 * Device dequantization exports: w_out [N,K] fp32 row-major, through the same
 * device unpacking code the GEMV kernels use.  Every value is exact (the
 * dequantized weights of these formats are exactly representable in fp32).
 * ------------------------------------------------------------------------- */
int dequant_int4_blockwise(const void* w_packed, const void* scales_f16, const void* zeros_u4,
                           float* w_out, int N, int K, int block_size, int layout, void* stream);
/* (layout selects how w_packed is read: canonical or B200_V1.) */

/* w_dsc NULL: coefficients decoded from the packed fields; else taken from the
 * plane.  layout WQ_LAYOUT_B200_V1 reads a wq_repack_q4k stream (w_dsc must
 * then be NULL). */
int dequant_q4k(const void* w_q4k, const void* w_dsc, float* w_out, int N, int K, int layout,
                void* stream);

/* mxfp4: w_out[n][k] = 2^(E - 127)·e2m1(q) exactly in fp32 (a value past the
 * fp32 range is ±inf; E = 255 gives NaN).  K % 32 == 0; w_packed and w_out
 * 16-byte aligned. */
int dequant_mxfp4(const void* w_packed, const void* scales_e8m0, float* w_out, int N, int K, void* stream);

/* ---------------------------------------------------------------------------
 * Row-split (tensor-parallel) layers: each GPU holds a run of W's rows and
 * computes those outputs; the all-gather of y is done by the GEMV's own
 * stores.  No counterpart on the pages (they run one GPU): this is the
 * N-split the hot-path scope table names for more than one GPU.
 * ------------------------------------------------------------------------- */

/* Rows [*n0, *n1) of rank `rank` of `world` for an N-row weight split in
 * units of `align` rows (16: whole B200_V1 bands), as evenly as possible
 * (the first N/align mod world ranks take one unit more; a rank may get
 * none, n0 == n1).  Host only.  Errors: WQ_ERR_ARG. */
int wq_tp_rows(int N, int world, int rank, int align, int* n0, int* n1);

/* y rows n_offset .. n_offset + N_shard - 1 of an int4 layer whose B200_V1
 * shard (rows n_offset.. of the full weight, repacked alone by
 * wq_repack_int4) is w_shard, stored into every one of the n_dsts (1..8)
 * buffers y_dsts[d] (a host array of device pointers), each a full [M][N_total]
 * fp16 output: this GPU's own y and, mapped into this process with
 * wq_ipc_open, the other GPUs' copies, so that when every rank's call has
 * finished each GPU holds all of y (the caller orders that with its own
 * barrier, e.g. stream synchronize + a host or NCCL barrier).  Runs the B200_V1
 * band kernel (blocks >= 128, K % 128 == 0); other columns are not touched.
 * x 16-byte aligned, destinations 2-byte aligned.  Errors: WQ_ERR_ARG,
 * WQ_ERR_ALIGN, WQ_ERR_UNSUPPORTED, WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int gemv_int4_tp(const void* x_f16, const void* w_shard, void* const* y_dsts, int n_dsts, int M, int N_shard, int K,
                 int block_size, int N_total, int n_offset, void* stream);

/* CUDA IPC for the destinations of gemv_int4_tp.  wq_ipc_handle: the 64-byte
 * handle of the allocation that holds dev_ptr (a pointer may sit inside a
 * larger allocation, e.g. one made by a caching allocator) and the byte
 * offset of dev_ptr in it.  wq_ipc_open: another process's (handle, offset)
 * mapped into this one (peer access enabled lazily), the pointer to the same
 * bytes.  wq_ipc_close: releases that mapping (same pointer and offset).
 * Errors: WQ_ERR_ARG, WQ_ERR_CUDA. */
int wq_ipc_handle(const void* dev_ptr, void* handle_out, unsigned long long* offset_out);
int wq_ipc_open(const void* handle, unsigned long long offset, void** dev_ptr_out);
int wq_ipc_close(void* dev_ptr, unsigned long long offset);

/* ---------------------------------------------------------------------------
 * int8-activation batched q4_K (minfer doc 62 "r59 — q4_K W_dsc plane", §3.2:
 * the MMQ dispatch arm quantizes the activations to int8 in a prepass and
 * runs an integer GEMM whose (chunk, row) pairs are rescaled by the §2.1
 * coefficients).  Numerically this is a different product from gemv_q4k: x is
 * replaced by its int8 quantization.
 * ------------------------------------------------------------------------- */

/* The q8 prepass.  For every token m and 32-element chunk c of x [M][K] fp16
 * (binary32, one rounding per operation): amax = max|x|, d = amax / 127,
 * q = x / d rounded to nearest, ties to even (0 when d = 0; |q| <= 127),
 * s = d·Σq.  Writes qa8 int8 [M][K] (token-major, wq_q8_bytes) and sda
 * float2 [K/32][Mp] = (d, s), Mp = M rounded up to 16, entries of tokens
 * M..Mp-1 zero (chunk-major, wq_q8_scale_bytes).  K % 32 == 0; every pointer
 * 16-byte aligned; x finite (the result for inf / NaN inputs is unspecified).
 * Errors: WQ_ERR_ARG, WQ_ERR_ALIGN, WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int quantize_q8(const void* x_f16, void* qa8, void* sda, int M, int K, void* stream);
size_t wq_q8_bytes(int M, int K);       /* M·K, 0 if invalid */
size_t wq_q8_scale_bytes(int M, int K); /* 8·(K/32)·Mp, 0 if invalid */

/* y[M,N] fp16 = Σ_c (d·sc)[n,c]·d[m,c]·I[m,n,c] + (−dmin·m)[n,c]·s[m,c],
 * I[m,n,c] = Σ_{k in chunk c} q4[n,k]·qa8[m,k] (exact), fp32 accumulation,
 * for canonical q4_K weights (w_q4k [N][K/256][144]) and the prepass output
 * (qa8, sda).  w_dsc (nullable): the W_dsc plane of the same weights, read
 * for the coefficients instead of decoding them (the results are bit-
 * identical).  tcgen05 kind::i8 GEMM.  K % 256 == 0; qa8, sda, w_q4k and
 * w_dsc 16-byte aligned, y 2-byte aligned.  WQ_FORCE_KERNEL other than "mmq"
 * returns WQ_ERR_UNSUPPORTED.  Errors: WQ_ERR_ARG, WQ_ERR_ALIGN,
 * WQ_ERR_UNSUPPORTED, WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int gemm_q4k_q8(const void* qa8, const void* sda, const void* w_q4k, const void* w_dsc, void* y_f16, int M, int N,
                int K, void* stream);

/* ---------------------------------------------------------------------------
 * Weight packing (load time).
 * ------------------------------------------------------------------------- */

/* Bytes of the int4 arrays (codes + scales + zero-points) for a layout; 0 for
 * invalid arguments. */
size_t wq_int4_bytes(int N, int K, int block_size, int layout);

/* Bytes of the canonical int4 code array ([N][K/2]); 0 if invalid. */
size_t wq_int4_codes_bytes(int N, int K, int layout);

/* Rewrite canonical int4 weights (codes [N][K/2], scales, zeros or NULL)
 * into layout `to_layout` at w_out (wq_int4_packed_bytes(N, K, block_size,
 * to_layout) bytes, device, must not overlap the sources).  Errors:
 * WQ_ERR_ARG (K % 128 != 0 or block_size < 32 for B200_V1), WQ_ERR_LAYOUT,
 * WQ_ERR_ALIGN, WQ_ERR_CUDA. */
int wq_repack_int4(const void* w_canonical, const void* scales_f16, const void* zeros_u4, void* w_out,
                   int N, int K, int block_size, int to_layout, void* stream);

/* Bytes of the buffer wq_repack_int4 writes (B200_V1), 0 if invalid. */
size_t wq_int4_packed_bytes(int N, int K, int block_size, int layout);

/* Rewrite two canonical int4 weights of the same shape (gate and up
 * projections: codes, scales, zero-points or NULL each) into the fused
 * B200_V1 gate-up stream at w_out (wq_int4_gate_up_packed_bytes bytes,
 * device): tile slot 2i holds tile i of the gate stream, slot 2i + 1 tile i
 * of the up stream.  block_size 128 or 256, K % 128 == 0.  Errors:
 * WQ_ERR_ARG, WQ_ERR_LAYOUT, WQ_ERR_ALIGN, WQ_ERR_CUDA. */
int wq_repack_int4_gate_up(const void* w_gate, const void* scales_gate, const void* zeros_gate,
                           const void* w_up, const void* scales_up, const void* zeros_up, void* w_out,
                           int N, int K, int block_size, int to_layout, void* stream);

/* Bytes of the fused gate-up stream (twice the B200_V1 stream), 0 if invalid. */
size_t wq_int4_gate_up_packed_bytes(int N, int K, int block_size, int layout);

/* Bytes of a q4_K tensor and of its W_dsc plane; 0 for invalid arguments. */
size_t wq_q4k_bytes(int N, int K);
size_t wq_q4k_dsc_bytes(int N, int K);

/* Bytes of the B200_V1 q4_K stream of an N × K tensor (layout must be
 * WQ_LAYOUT_B200_V1), 0 if invalid. */
size_t wq_q4k_packed_bytes(int N, int K, int layout);

/* Rewrite canonical q4_K super-blocks (N·(K/256)·144 bytes, device) into the
 * B200_V1 q4_K stream at w_out (wq_q4k_packed_bytes(N, K, to_layout) bytes,
 * device, must not overlap the source).  Errors: WQ_ERR_ARG (K % 256 != 0),
 * WQ_ERR_LAYOUT (to_layout is not WQ_LAYOUT_B200_V1), WQ_ERR_ALIGN,
 * WQ_ERR_CUDA. */
int wq_repack_q4k(const void* w_q4k, void* w_out, int N, int K, int to_layout, void* stream);

/* Build the W_dsc plane on the host (minfer doc 62, §2.2-§2.3): one IEEE fp32
 * multiply per coefficient and an exact negation, no contraction.
 * w_q4k_host: N·(K/256)·144 bytes; out_host: wq_q4k_dsc_bytes(N, K) bytes. */
int wq_build_q4k_dsc(const void* w_q4k_host, int N, int K, void* out_host);

/* The same plane built on the device (bit-identical to the host builder). */
int wq_build_q4k_dsc_device(const void* w_q4k, void* out, int N, int K, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 * ------------------------------------------------------------------------- */
const char* wq_last_error(void);   /* message of the last failure on this thread */
const char* wq_last_kernel(void);  /* liveness label of the last launch on this thread */
int wq_layout_version(void);       /* newest layout version this library reads (WQ_LAYOUT_B200_V1) */
const char* wq_build_info(void);   /* "sm_100a ..." build description */

/* Synchronizes the current device, then reads and clears the device-side
 * error word that bounded waits set when they give up.  Returns WQ_OK or
 * WQ_ERR_TIMEOUT (or WQ_ERR_CUDA if the synchronization itself fails). */
int wq_device_status(void);

/* Test hook for the failure path of bounded device waits (no counterpart on
 * the pages; it exists so the timeout status can be tested without faulting a
 * GPU).  Enqueues one tiny kernel on `stream` whose single thread waits on an
 * mbarrier that nothing arrives at, with no copy in flight, and gives up after
 * limit_ns nanoseconds (1e3 .. 1e9), recording the timeout in the device
 * error word exactly as a real wait that gives up does; the kernel then
 * returns.  The next wq_device_status() reports WQ_ERR_TIMEOUT once.
 * Errors: WQ_ERR_ARG (limit out of range), WQ_ERR_DEVICE, WQ_ERR_CUDA. */
int wq_test_expire_wait(unsigned long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
