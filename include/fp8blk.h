/*
 * fp8blk -- FP8 (E4M3) blockwise-scaled quantisation and GEMM for NVIDIA B200 (sm_100a).
 *
 * The operations follow the Puro-2B FP8 recipe as described on these pages:
 *   [EXPL]   "用 RTX 5090 花 $7000 训练 2B 大模型：Puro-2B 低成本预训练技术解析"
 *            (hankli.space): section "Blackwell 的 FP8 Tensor Core" (E4M3 =
 *            float8_e4m3fn, 4 exponent / 3 mantissa bits, max 448), section
 *            "核心挑战：Scale Factor 管理" (scale = amax/448 floored at 1e-12,
 *            codes = cast(clamp(x/scale, +-448)); the layer's output is the
 *            matmul of the dequantised operands) and section "常见错误：直接转换
 *            而不加 Scale" (the same scale rule without the floor).
 *   [DIGEST] "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090"
 *            (AI Papers Daily): "工作参考价值" bullet 2 and "方法关键点" bullet
 *            "FP8 blockwise 混合精度": activations in 1-D groups of 128,
 *            weights in 128x128 blocks, linear-layer GEMMs in E4M3.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or keeps a pointer after the call returns.
 *  - Matrices are row-major; "[R][C]" means C contiguous elements per row.
 *    bf16 inputs are raw bfloat16 bit patterns (uint16).  E4M3 codes are
 *    float8_e4m3fn bytes.  Scales are IEEE binary32.
 *  - Every dimension must be a positive multiple of 128 (FP8BLK_ERR_SHAPE).
 *    Pointers must be 16-byte aligned and leading dimensions must give
 *    16-byte aligned rows (FP8BLK_ERR_ALIGN).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; argument errors are returned
 *    before anything is enqueued; a launch failure returns FP8BLK_ERR_LAUNCH.
 *  - Inputs must be finite; NaN or Inf in an input gives unspecified codes.
 *  - The quantisers are exact: codes and scales equal, bit for bit,
 *        s = max(fl32(amax / 448), fl32(1e-12))
 *        q = E4M3_round_nearest_even(clamp(fl32(x / s), -448, 448))
 *    with amax the largest |x| of the group and x / s a correctly rounded
 *    binary32 division.  The sign of zero is kept (-0 -> 0x80).
 *  - Device-side waits are bounded in time.  A wait that expires makes the
 *    kernel stop early, leaving its outputs unspecified, and records
 *    FP8BLK_ERR_TIMEOUT in a device error word read by
 *    fp8blk_get_device_error().
 *  - Environment variables, read at every call (tuning and tests only; the
 *    defaults are the measured best on B200):
 *      FP8BLK_WAIT_TIMEOUT_MS     bound of each device-side wait (default 4000)
 *      FP8BLK_PDL=1               launch with programmatic dependent launch
 *      FP8BLK_GEMM_BLOCK_N        128 or 256: force the GEMM tile width
 *      FP8BLK_GEMM_PAIR           1: 256x256 tiles on CTA pairs wherever M and
 *                                 N are multiples of 256; 0: never (default)
 *      FP8BLK_GEMM_GROUP_M        M-blocks per group of the GEMM tile order
 *      FP8BLK_GEMM_SPLITK=0       fp8blk_gemm_splitk_count returns 1 (no split)
 *      FP8BLK_GEMM_MAX_CTAS       at most this many GEMM CTAs (one per SM), so
 *                                 that concurrent work on other streams finds
 *                                 free SMs (default: one per SM)
 *      FP8BLK_QUANT_MAX_CTAS      the same for the quantisers (default: as many
 *                                 as fit, two per SM)
 *      FP8BLK_TEST_INJECT_STALL=1 tests only: one wait of the next launch
 *                                 never completes, so that the bounded-wait
 *                                 error path runs
 */
#ifndef FP8BLK_H
#define FP8BLK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8BLK_OK = 0,
  FP8BLK_ERR_INVALID_ARG = 1,        /* NULL pointer where one is required, bad mode/layout, ld too small */
  FP8BLK_ERR_SHAPE = 2,              /* a dimension <= 0 or not a multiple of 128 */
  FP8BLK_ERR_ALIGN = 3,              /* a pointer or row stride not 16-byte aligned */
  FP8BLK_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 (B200, sm_100a) */
  FP8BLK_ERR_LAUNCH = 5,             /* the CUDA launch (or a CUDA call it needs) failed */
  FP8BLK_ERR_TIMEOUT = 6,            /* a bounded device-side wait expired (reported by fp8blk_get_device_error) */
  FP8BLK_ERR_CUDA = 7                /* a CUDA runtime call outside a launch failed */
} fp8blk_status;

typedef enum {
  FP8BLK_ROWWISE = 1,   /* 1x128 groups along the contiguous (feature) dimension */
  FP8BLK_COLWISE_T = 2, /* 1x128 groups along rows (tokens); codes written transposed */
  FP8BLK_BOTH = 3,      /* both of the above from one read of the input */
  FP8BLK_E5M2 = 4       /* OR-ed into a mode: E5M2 codes instead of E4M3 (gradients) */
} fp8blk_act_mode;

typedef enum {
  FP8BLK_FWD = 0,   /* B scales per 128x128 block: sb[N/128][K/128] */
  FP8BLK_DGRAD = 1, /* same operand format as FWD (B = transposed weight) */
  FP8BLK_WGRAD = 2  /* B scales per row and K-block: sb[K/128][N] */
} fp8blk_layout;

/* OR-ed into a layout: operand A (or B) holds E5M2 codes instead of E4M3;
 * FP8BLK_OUT_F32: d receives the fp32 sums unrounded (for a partial result
 * that is summed further, such as one rank's share of a data-parallel weight
 * gradient; see fp8blk_round_f32_to_bf16). */
typedef enum {
  FP8BLK_A_E5M2 = 8,
  FP8BLK_B_E5M2 = 16,
  FP8BLK_OUT_F32 = 32
} fp8blk_operand_format;

/*
 * Activation quantisation, 1x128 groups ([DIGEST] "激活 1D 128"; scale and
 * cast rule from [EXPL] "核心挑战：Scale Factor 管理").
 *
 *   x      [rows][ldx] bf16, the first `cols` columns of each row are used.
 *   mode   FP8BLK_ROWWISE, FP8BLK_COLWISE_T or FP8BLK_BOTH, optionally OR-ed
 *          with FP8BLK_E5M2: E5M2 codes ([EXPL] "Blackwell 的 FP8 Tensor
 *          Core": 5 exponent bits, 2 mantissa bits, max 57344, the format for
 *          gradients) with scale = max(fl32(amax / 57344), fl32(1e-12)) and the
 *          value clamped to +-57344 before the cast; otherwise E4M3 as below.
 *   ROWWISE outputs (required for ROWWISE and BOTH, else ignored):
 *     q_row  [rows][cols] E4M3 codes, group = 128 consecutive columns of a row
 *     s_row  [cols/128][rows] fp32, s_row[g][r] = scale of row r, group g
 *   COLWISE_T outputs (required for COLWISE_T and BOTH, else ignored):
 *     q_colT [cols][rows] E4M3 codes = the codes of x^T, group = 128
 *            consecutive rows (tokens) of one column
 *     s_colT [rows/128][cols] fp32, s_colT[g][c] = scale of column c, group g
 *   The forward and data-gradient GEMMs take (q_row, s_row) as operand A;
 *   the weight-gradient GEMM takes (q_colT, s_colT) of the output gradient as
 *   A and of the layer input as B.
 */
fp8blk_status fp8blk_quantize_act_1x128(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                        int mode, uint8_t* q_row, float* s_row,
                                        uint8_t* q_colT, float* s_colT, void* stream);

/*
 * Weight quantisation, 128x128 blocks ([DIGEST] "权重 2D 128x128").
 *   w  [n][ldw] bf16 (first k columns used)  ->  q [n][k] E4M3,  s [n/128][k/128] fp32.
 * The forward GEMM takes (q, s) as operand B.
 */
fp8blk_status fp8blk_quantize_weight_128x128(const void* w, int64_t n, int64_t k, int64_t ldw,
                                             uint8_t* q, float* s, void* stream);

/*
 * The same 128x128 blocks (so the same scales and codes), written transposed:
 *   w  [n][ldw] bf16  ->  qT [k][n] E4M3,  sT [k/128][n/128] fp32.
 * qT[j][i] == q[i][j] and sT[b][a] == s[a][b] for the outputs of
 * fp8blk_quantize_weight_128x128.  The data-gradient GEMM
 * dX = dY . W takes (qT, sT) as operand B.
 */
fp8blk_status fp8blk_quantize_weight_128x128_t(const void* w, int64_t n, int64_t k, int64_t ldw,
                                               uint8_t* qT, float* sT, void* stream);

/*
 * Both of the above from one read of w (a training step needs both layouts:
 * (q, s) for the forward GEMM, (qT, sT) for the data-gradient GEMM).  The
 * outputs are bitwise those of the two separate calls.  Alignment and
 * argument errors as for the separate calls; all four outputs are required.
 */
fp8blk_status fp8blk_quantize_weight_128x128_both(const void* w, int64_t n, int64_t k, int64_t ldw,
                                                  uint8_t* q, float* s, uint8_t* qT, float* sT,
                                                  void* stream);

/*
 * The weights of a layer (or any set of weights) quantised in one launch:
 * for each entry, exactly the outputs of fp8blk_quantize_weight_128x128_both
 * on that weight.  One launch streams all weights' tiles through the
 * persistent CTAs, so the small weights do not each pay a launch, a first
 * tile and a last round of their own.
 *   weights  host array of `count` descriptors (read during the call only);
 *            every field as for fp8blk_quantize_weight_128x128_both, all four
 *            outputs required; the weights' buffers must not overlap each
 *            other's outputs.
 *   count    1 .. FP8BLK_MAX_WEIGHTS.
 * Errors: those of fp8blk_quantize_weight_128x128_both for any entry (the
 * first failing entry decides), FP8BLK_ERR_INVALID_ARG for a null array or a
 * count out of range.  Nothing is launched when any entry is invalid.
 */
#define FP8BLK_MAX_WEIGHTS 8
typedef struct {
  const void* w;   /* [n][ldw] bf16 */
  int64_t n, k, ldw;
  uint8_t* q;      /* [n][k] E4M3 */
  float* s;        /* [n/128][k/128] */
  uint8_t* qT;     /* [k][n] E4M3 */
  float* sT;       /* [k/128][n/128] */
} fp8blk_weight_128x128;

fp8blk_status fp8blk_quantize_weights_128x128_both(const fp8blk_weight_128x128* weights, int count,
                                                   void* stream);

/*
 * Blockwise-scaled FP8 GEMM with bf16 output ([EXPL] "核心挑战：Scale Factor
 * 管理": the output is linear(x_fp8 * x_scale, w_fp8 * w_scale); [DIGEST]
 * "方法关键点": the linear-layer GEMMs run in E4M3):
 *
 *   D[m][n] = bf16( sum over K-blocks kb of  sa(m,kb) * sb(n,kb) * P_kb[m][n] ),
 *   P_kb[m][n] = sum_{k in kb} a[m][k] * b[n][k]   (fp32 accumulation on the tensor cores)
 *
 *   a   [M][K] E4M3 codes (K contiguous),  sa [K/128][M] fp32 (per row, per K-block)
 *   b   [N][K] E4M3 codes (K contiguous)
 *   layout may be OR-ed with FP8BLK_A_E5M2 and/or FP8BLK_B_E5M2 when that
 *   operand holds E5M2 codes (E5M2 gradients: DGRAD and WGRAD take dY as A).
 *   sb  FWD / DGRAD: [N/128][K/128] fp32 (per 128x128 block)
 *       WGRAD      : [K/128][N] fp32     (per row of b, per K-block)
 *   d   [M][ldd] bf16 output, ldd >= N, ldd % 16 == 0, d 32-byte aligned;
 *       with FP8BLK_OUT_F32 in layout: fp32 output, ldd % 8 == 0 (the sums
 *       are stored without the bf16 rounding).
 *
 * Operands per pass of a linear layer Y = X . W^T (X [T][in], W [out][in]):
 *   FWD   : a = X rowwise,      b = W (128x128),           d = Y  [T][out]
 *   DGRAD : a = dY rowwise,     b = W transposed (128x128), d = dX [T][in]
 *   WGRAD : a = dY colwise_T,   b = X colwise_T,            d = dW [out][in]
 * The result is accumulated in fp32 and rounded once to bf16; it is not
 * bitwise reproducible against another summation order.
 */
fp8blk_status fp8blk_gemm(int layout, int64_t M, int64_t N, int64_t K,
                          const uint8_t* a, const float* sa, const uint8_t* b, const float* sb,
                          void* d, int64_t ldd, void* stream);

/*
 * The same GEMM with split-K, for shapes whose output tiles leave SMs idle:
 * with fewer tiles than SMs (the weight gradient of a narrow layer: few
 * tiles, long K) every tile is split; with more, the tiles of the last,
 * partial round of the SMs (tiles mod SMs of them) are, so that their units
 * fill that round.  The K-blocks of a split tile are divided among
 * `splits` work units; unit s sums its contiguous range of K-blocks (the same
 * per-K-block promotion as fp8blk_gemm) into an fp32 partial tile in
 * `workspace`, and a second kernel adds the partials in the order s = 0, 1,
 * ... in fp32 and rounds the total once to bf16 (or stores it as fp32 with
 * FP8BLK_OUT_F32).  The result is deterministic; it differs from
 * fp8blk_gemm's only by the order of the fp32 additions in the split tiles.
 *   splits      1 .. K/128; 1 runs fp8blk_gemm (workspace unused).
 *   workspace   device memory of at least
 *               fp8blk_gemm_splitk_workspace_bytes(layout, M, N, K, splits) bytes, 16-byte
 *               aligned, owned by the caller; overwritten; it must not overlap
 *               any operand or d, and must stay untouched until the call's
 *               kernels have run (stream order).
 * Errors as fp8blk_gemm; FP8BLK_ERR_INVALID_ARG for a split count out of
 * range or a missing or short workspace, FP8BLK_ERR_ALIGN for an unaligned
 * workspace (its size is checked after fp8blk_gemm's checks, on the device).
 */
fp8blk_status fp8blk_gemm_splitk(int layout, int64_t M, int64_t N, int64_t K,
                                 const uint8_t* a, const float* sa, const uint8_t* b, const float* sb,
                                 void* d, int64_t ldd, int splits, float* workspace,
                                 int64_t workspace_bytes, void* stream);

/*
 * Bytes of split-K workspace fp8blk_gemm_splitk needs for this GEMM and split
 * count on the current device: (split tiles) x splits x 128 x (tile width) x 4
 * (the split tiles: all of them with fewer tiles than SMs, else the last
 * round's tiles mod SMs; never more than splits * M * N * 4).  0 when splits == 1, -1 for an invalid
 * layout, shape or split count or an unsupported device.
 */
int64_t fp8blk_gemm_splitk_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int splits);

/*
 * The split count the library uses well for this GEMM shape on the current
 * device.  With fewer output tiles than SMs (all tiles are split): the count
 * (2 to 4, each unit keeping at least 16 K-blocks) whose units shorten the
 * run by at least 20% in whole-tile waves, else 1.  With more (only the tiles
 * of the last, partial round of the SMs are split): the largest count up to 8
 * whose units fit beside each other on the SMs with at least 12 K-blocks
 * each, else 1.  0 for an invalid layout or shape or an unsupported device.
 */
int fp8blk_gemm_splitk_count(int layout, int64_t M, int64_t N, int64_t K);

/*
 * Per-tensor delayed scaling ([EXPL] "核心挑战：Scale Factor 管理", FP8Linear):
 * one amax buffer per tensor (the caller initialises it to 1), updated from
 * the tensor's current max |x| by an exponential moving average before the
 * tensor is quantised with one scale.
 *
 * fp8blk_amax_ema: amax <- RN(RN(amax * RN32(0.99)) + RN(max|x| * RN32(1 - 0.99)))
 *   (binary32), then scale <- max(amax / 448, 1e-12) (correctly rounded).
 *   x          [rows][ldx] bf16, the first cols columns of each row are used.
 *   amax       device float, read and written (the EMA state).
 *   scale      device float, written.
 *   workspace  device scratch of at least fp8blk_amax_ema_workspace_bytes(rows)
 *              bytes (16-byte aligned), fully rewritten by every call, owned by
 *              the caller; two calls may share it only if they are ordered on
 *              one stream.  Too small: FP8BLK_ERR_INVALID_ARG.
 */
fp8blk_status fp8blk_amax_ema(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax, float* scale,
                              void* workspace, int64_t workspace_bytes, void* stream);
int64_t fp8blk_amax_ema_workspace_bytes(int64_t rows);

/*
 * fp8blk_amax_ema without a caller workspace and without allocating: the same
 * two kernels and the same result bits, the partial maxima kept in a fixed
 * 32 KiB device array inside this library.  The pages have no counterpart of
 * this entry point; it serves callers that must not allocate (an allocator
 * being set up, a captured graph built without a memory pool).
 *   Rows above FP8BLK_AMAX_EMA_STATIC_MAX_ROWS: FP8BLK_ERR_SHAPE; other
 *   argument errors as for fp8blk_amax_ema.
 *   Nothing needs to start at zero: each call rewrites every partial it reads.
 *   The array is one per device and per process: calls on one device must be
 *   ordered (one stream, or events); two in flight at once on different
 *   streams race on it and may return a wrong amax.
 *   The first call on a device looks up the array's address
 *   (cudaGetSymbolAddress; a failure returns FP8BLK_ERR_CUDA) and caches it:
 *   make that call before capturing a CUDA graph that contains this entry
 *   point.  Later calls look nothing up and allocate nothing: the device
 *   check and the two kernel launches.
 */
#define FP8BLK_AMAX_EMA_STATIC_MAX_ROWS 65536
fp8blk_status fp8blk_amax_ema_static(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax,
                                     float* scale, void* stream);

/*
 * Quantise a whole tensor with the one scale *scale (device float, e.g. from
 * fp8blk_amax_ema): q = E4M3(RN(clamp(x / scale, -448, 448))).  A stale amax
 * may put |x / scale| far above 448: those values saturate to +-448.
 *   x [rows][ldx] bf16 -> q [rows][cols] E4M3.
 */
fp8blk_status fp8blk_quantize_tensor(const void* x, int64_t rows, int64_t cols, int64_t ldx, const float* scale,
                                     uint8_t* q, void* stream);

/*
 * GEMM with one scale per operand ([EXPL] FP8Linear.forward: the product of
 * the dequantised operands):  D[m][n] = bf16( *sa * *sb * sum_k a[m][k] b[n][k] ),
 * the sum accumulated in fp32 on the tensor cores over the whole K loop.
 *   a [M][K] E4M3, b [N][K] E4M3 (both K-major), sa / sb device floats,
 *   d [M][ldd] bf16 (ldd % 16 == 0, d 32-byte aligned).  Errors as for fp8blk_gemm.
 */
fp8blk_status fp8blk_gemm_tensor_scaled(int64_t M, int64_t N, int64_t K, const uint8_t* a, const float* sa,
                                        const uint8_t* b, const float* sb, void* d, int64_t ldd, void* stream);

/*
 * y[i] = bf16(x[i]), round to nearest even, for 0 <= i < n: the single
 * rounding of a sum of fp32 partial results.  Used for the data-parallel
 * weight gradient: the pages' training run sums gradients across GPUs with
 * an all-reduce ("小团队也能预训练！普罗2B" (66bd.net), the paragraph on the
 * 24-GPU AllReduce over GPUDirect RDMA); each rank's WGRAD GEMM writes its
 * partial dW in fp32 (FP8BLK_OUT_F32), the partials are summed in fp32 by the
 * all-reduce, and this call rounds the sum to bf16 once.
 *   x  [n] fp32 device array, y [n] bf16 device array, both 16-byte aligned;
 *   n > 0 (else FP8BLK_ERR_SHAPE).  x and y must not overlap.
 */
fp8blk_status fp8blk_round_f32_to_bf16(const float* x, int64_t n, void* y, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * device the stream belongs to (the current device for the default streams).  Returns FP8BLK_OK, FP8BLK_ERR_TIMEOUT if a kernel's
 * bounded wait expired since the last call, or FP8BLK_ERR_CUDA if the
 * synchronisation itself failed.
 */
fp8blk_status fp8blk_get_device_error(void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char* fp8blk_status_string(fp8blk_status status);

/* Library version as major*10000 + minor*100 + patch. */
int fp8blk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BLK_H */
