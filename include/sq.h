/*
 * sq.h -- C ABI of the separated-quantization decode linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * The method (Chinese-language web page "1-bit量化不是玄学，以往掉点是机制问题",
 * m.lqnn.cn/news/241359, sections 2.1-2.3, 3.3, 5.2, 5.3 and 6.2):
 *   W ~ alpha_r * sign(W) + W_res        one 1-bit sign trunk, one scale per row
 *   W_res = W - alpha_r * sign(W)       re-quantized to INT8 (groups along K)
 *   x -> fp32 outlier channels + INT8 per-token codes on the other channels
 *   y = (trunk product by bit operations) + (residual integer product)
 *       + (outlier channels at full precision), all in one kernel.
 * The symmetric INT8 quantizer follows the "对称量化以零为中心" (absmax) section of
 * the visual guide to LLM quantization (puppylpg.github.io) and the divide
 * convention s = absmax/127, q = round(x/s) of the 2048ai.net explainer,
 * section 三.1; the sign of zero follows the BitNet "权重量化" paragraph of the
 * visual guide (non-negative -> +1).
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers owned by the caller, unless stated.
 *    The library never allocates device memory; sizes are queryable.
 *  - Every call is asynchronous on the caller's stream ("stream" is a
 *    cudaStream_t; NULL = the legacy default stream).  The return value only
 *    covers host-side validation and the launch itself.
 *  - Device-side findings (non-finite input, a wait that ran out) are written
 *    to the optional caller-owned int32 word "dev_status" (device memory): it
 *    is left untouched on success and set to a sq_status code otherwise.
 *  - Pointers must be 16-byte aligned (else SQ_ERR_ALIGN).
 *  - The current device must be an sm_100 (B200-class) GPU, else
 *    SQ_ERR_UNSUPPORTED_DEVICE.  There is no CPU fallback.
 *  - Calls on one stream are ordered; calls that share output or workspace
 *    buffers on different streams must be ordered by the caller.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,        /* NULL pointer, bad enum, unsorted index list */
  SQ_ERR_SHAPE = 2,              /* size out of the supported range */
  SQ_ERR_ALIGN = 3,              /* a pointer is not 16-byte aligned */
  SQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 */
  SQ_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  SQ_ERR_NONFINITE = 6,          /* (device status) NaN or Inf in an input */
  SQ_ERR_TIMEOUT = 7,            /* (device status) a bounded wait ran out */
  SQ_ERR_WORKSPACE = 8           /* workspace missing or too small */
} sq_status;

/* Launch flags (bit set). */
#define SQ_LAUNCH_PDL 1u
#define SQ_TRUNK_ONLY 2u
/* SQ_TRUNK_ONLY (sq_linear, sq_quantize_linear, sq_linear_noalloc; weights in
 * SQ_LAYOUT_TILES or SQ_LAYOUT_TILES_SPARSE only, else SQ_ERR_INVALID_ARG):
 * the residual path is
 * skipped (m.lqnn.cn section 3.3: the 1-bit trunk first, the residual added
 * on demand; a request that tolerates a rougher answer skips it).  The
 * residual codes and scales are not read:
 *   y_tr = sx_t * alpha_r * T_tr + sum_i Wt_{r,idx_i} * x_out_ti,
 *   Wt_rj = m_rj * alpha_r * (2 b_rj - 1)
 * (outlier channels take the trunk weight).  Not accepted by
 * sq_linear_accumulators. */
/* SQ_LAUNCH_PDL: launch with programmatic dependent launch.  The kernel may
 * start while the previous kernel in the stream is still running: it begins
 * streaming the packed weights and reads the outlier index list (both fixed
 * once a layer is set up) at once, and reads every other input and writes
 * every output only after the previous kernel has completed.  Set it only if
 * no earlier work still in flight on the stream writes the packed weights or
 * the index list. */

/* Packed-weight layouts (sq_packed_weight.layout). */
#define SQ_LAYOUT_ROWS 0
#define SQ_LAYOUT_TILES 1
#define SQ_LAYOUT_TILES_SPARSE 2
#define SQ_LAYOUT_TILES_ASYM 3

/*
 * Packed weight of one linear layer (N output rows, K input channels).
 * The content is the same in both layouts: sign bit b = [W[r][j] >= 0] (so
 * both zeros give 1), trunk mask bit, per-row trunk scale alpha, residual
 * code in [-127, 127] and residual scale of group g = channels [g*G, g*G+G).
 * Pads (bits, codes, scales, alpha) are 0.
 *
 * SQ_LAYOUT_ROWS (any G; decoded on the CUDA cores), row-major:
 *   sign_bits [N][sign_stride] u32  bit (j % 32) of word (j / 32) = channel j
 *   mask_bits [N][sign_stride] u32  same bit layout; NULL = full trunk
 *   alpha     [roundup(N,8)]   f32
 *   res_q     [N][res_stride]  i8
 *   res_scale [N][scale_stride] f32
 *   sign_stride = roundup(ceil(K/32), 4), res_stride = roundup(K, 16),
 *   scale_stride = roundup(ceil(K/G), 4).
 *
 * SQ_LAYOUT_TILES (G = 128 only; decoded on the tensor cores): the order in
 * which the decode kernel streams the weight.  Rows are padded to
 * N16 = roundup(N, 16) and channels to K128 = roundup(K, 128); tile
 * t = rb*tpr + g (tpr = K128/128) covers rows [16rb, 16rb+16) and channels
 * [128g, 128g+128).  Within a tile, lane L = 4*gid + q owns rows
 * r0 = 16rb + gid, r1 = r0 + 8 and channels 128g + 32q + j (j = 0..31);
 * word w = j/4 holds channels 4w..4w+3.
 *   res_q     tile t at byte 2048*t, lane L at +64*L: four 16-byte groups
 *             m = 0..3 of words {r0 w=2m, r1 w=2m, r0 w=2m+1, r1 w=2m+1}
 *   sign_bits tile t at word 64*t; lane L: word 2L (row r0), 2L+1 (row r1);
 *             channel j of the lane's 32 at bit 8*(j%4) + j/4
 *   mask_bits same as sign_bits; NULL = full trunk
 *   res_scale tile t at float 16*t, one per row of the row block
 *   alpha     [N16] f32
 *   sign_stride = K128/32, res_stride = K128, scale_stride = K128/128
 *   (the padded row lengths).  K <= 131072.
 *
 * SQ_LAYOUT_TILES_SPARSE (G = 128 only; written by sq_decompose_pack_sparse):
 * SQ_LAYOUT_TILES with a sparse residual (m.lqnn.cn section 3.3: residual
 * entries near zero are dropped and the rest stored sparsely).  Two arrays
 * more, and res_q holds each tile's kept codes only:
 *   keep_bits same shape and bit order as sign_bits: 1 = the residual entry
 *             is kept, 0 = dropped (its code is 0)
 *   res_q     tile t's slot of 2048 bytes at byte 2048*t holds the tile's
 *             kept codes, packed: lane L = 0..31 in order, within a lane row
 *             r0's 32 channels then row r1's, ascending channel; zero padded
 *             to a multiple of 16 bytes; the rest of the slot is unused
 *   res_bytes [T] i32, T = (N16/16)*(K128/128): the padded byte count of
 *             each tile's kept codes (what the decode kernel reads)
 * Every other array is that of SQ_LAYOUT_TILES.
 *
 * SQ_LAYOUT_TILES_ASYM (G = 128 only): SQ_LAYOUT_TILES with an asymmetric
 * residual (m.lqnn.cn section 2 pitfalls: the residual gets its own min/max,
 * scale and zero-point; the asymmetric quantizer of the 2048ai.net
 * explainer): codes in [-128, 127] and one more array,
 *   res_zero  [tile][16] i32, indexed like res_scale: the zero-point z_g of
 *             each (row, group); the dequantized residual is s_g*(q - z_g)
 * Every other array is that of SQ_LAYOUT_TILES.
 *
 * The arrays may live in one allocation carved by sq_packed_view().
 */
typedef struct {
  int32_t N, K, group_size;  /* group_size G: 32, 64 or 128 */
  int32_t layout;            /* SQ_LAYOUT_ROWS, SQ_LAYOUT_TILES, _TILES_SPARSE or _TILES_ASYM */
  int32_t sign_stride;       /* u32 words per row of sign_bits / mask_bits */
  int32_t res_stride;        /* bytes per row of res_q */
  int32_t scale_stride;      /* floats per row of res_scale */
  uint32_t *sign_bits;
  uint32_t *mask_bits;       /* NULL = full trunk */
  float *alpha;
  int8_t *res_q;
  float *res_scale;
  uint32_t *keep_bits;       /* SQ_LAYOUT_TILES_SPARSE only, else NULL */
  int32_t *res_bytes;        /* SQ_LAYOUT_TILES_SPARSE only, else NULL */
  int32_t *res_zero;         /* SQ_LAYOUT_TILES_ASYM only, else NULL */
} sq_packed_weight;

/* Human-readable name of a status code (static string, never NULL). */
const char *sq_status_string(sq_status s);

/* Checks that the current device is sm_100.  SQ_OK or SQ_ERR_UNSUPPORTED_DEVICE. */
sq_status sq_device_check(void);

/* Bytes of one allocation that holds a packed weight of this shape and
 * layout (the five arrays, each 256-byte aligned inside it).  0 for an
 * unsupported shape, group size or layout. */
size_t sq_packed_bytes(int32_t N, int32_t K, int32_t group_size, int32_t with_mask,
                       int32_t layout);

/* Fills *out with the strides and with pointers into "base" (device memory of
 * at least sq_packed_bytes() bytes, 256-byte aligned).  Host-only; no device
 * work.  with_mask = 0 leaves mask_bits NULL. */
sq_status sq_packed_view(void *base, int32_t N, int32_t K, int32_t group_size,
                         int32_t with_mask, int32_t layout, sq_packed_weight *out);

/*
 * Offline decomposition ("分离阶段（离线完成）", m.lqnn.cn section 5.3; the split of
 * section 2.1; the per-row threshold of sections 5.2 and 6.2).
 *   W             [N][K] f32 row-major, device, read only
 *   trunk_percent < 0: every element is in the trunk (out->mask_bits may be
 *                 NULL).  1..100: per row, tau_r = the ceil(P*K/100)-th
 *                 smallest |W[r][j]| (nearest rank) and the trunk is
 *                 |W| > tau_r (out->mask_bits must be set).
 *   out           strides and pointers as from sq_packed_view(); written in
 *                 full, pads included.
 * alpha_r = float(S / cnt), S the binary64 sum of |W| over the trunk members
 * in ascending channel order, cnt their number (0 -> alpha 0).  Residual
 * r = double(W) - m*(+-alpha) in binary64; group scale s = float(absmax/127);
 * code = clip(round_half_away(r / s), +-127) with a binary64 quotient (s == 0
 * gives 0).  Into SQ_LAYOUT_TILES_ASYM the residual groups are asymmetric:
 * lo, hi = the group's min and max of r, s = float((hi - lo) / 255),
 * z = round_half_away(-lo / s - 128), code = clip(round_half_away(r / s + z),
 * -128, 127), all in binary64 (s == 0 gives z = 0 and codes 0).
 * Non-finite W sets SQ_ERR_NONFINITE in dev_status.
 */
sq_status sq_decompose_pack(const float *W, int32_t N, int32_t K, int32_t trunk_percent,
                            const sq_packed_weight *out, int32_t *dev_status, void *stream);

/*
 * sq_decompose_pack with a sparse residual, into SQ_LAYOUT_TILES_SPARSE
 * (m.lqnn.cn section 3.3: a small threshold zeroes the residual entries
 * near zero, typically 50-70 % of them, and the residual is stored sparsely;
 * the page gives no threshold rule).  Trunk, alpha and residual r as in
 * sq_decompose_pack; then, per row, theta_r = the ceil(Ps*K/100)-th smallest
 * |r| over the row's K channels (binary64; nearest rank, as the trunk
 * threshold) and an entry is kept iff |r| > theta_r (ties dropped); group
 * scales come from the kept entries only (s = float(max kept |r| / 127),
 * 0 for a group with none kept) and a kept entry's code is
 * clip(round_half_away(r / s), +-127).
 *   residual_percent  Ps, 1..99
 *   out               strides and pointers as from sq_packed_view() with
 *                     layout SQ_LAYOUT_TILES_SPARSE; written in full.
 * Non-finite W sets SQ_ERR_NONFINITE in dev_status.
 */
sq_status sq_decompose_pack_sparse(const float *W, int32_t N, int32_t K, int32_t trunk_percent,
                                   int32_t residual_percent, const sq_packed_weight *out,
                                   int32_t *dev_status, void *stream);

/*
 * The per-layer fallback measure (m.lqnn.cn section 2.3, last paragraph: a
 * layer that gains nothing from the split falls back to plain 8-bit).
 *   W        [N][K] f32, device: the weight that `w` was decomposed from
 *   w        packed weight of W (any layout but SQ_LAYOUT_TILES_SPARSE)
 *   err      device, 2 doubles out:
 *            err[0] = sum_r sum_j (W_rj - What_rj)^2 for w, What its
 *                     dequantized weight (trunk + residual);
 *            err[1] = the same for plain symmetric INT8 groups of W of w's
 *                     group size (no trunk): What = s_g*Q(W, s_g),
 *                     s_g = float(absmax_g |W| / 127);
 *            each binary64, channels ascending within a row, rows in order.
 *   scratch  device, sq_residual_errors_scratch_bytes(N) bytes
 * The rule (this library's reading of the page): the layer falls back --
 * it is packed with trunk_percent = 100, an empty trunk, i.e. plain INT8
 * groups of W -- when err[1] <= err[0], that is when the split does not
 * reconstruct W strictly better.
 */
size_t sq_residual_errors_scratch_bytes(int32_t N);
sq_status sq_residual_errors(const float *W, const sq_packed_weight *w, double *err,
                             void *scratch, size_t scratch_bytes, int32_t *dev_status,
                             void *stream);

/*
 * The split with the per-layer fallback applied (the rule above): decomposes
 * W into *out with trunk_percent (as sq_decompose_pack), measures both
 * errors and, when err[1] <= err[0], decomposes W again with
 * trunk_percent = 100 (an empty trunk: plain INT8 groups of W).
 *   out       packed weight with a mask array (layout SQ_LAYOUT_ROWS,
 *             SQ_LAYOUT_TILES or SQ_LAYOUT_TILES_ASYM); on return
 *             out->mask_bits is set to NULL when the split was kept with a
 *             full trunk (trunk_percent < 0), whose all-ones mask the decode
 *             kernels need not read (the array stays in the caller's buffer)
 *   scratch   device, sq_residual_errors_scratch_bytes(N) + 256 bytes
 *   fell_back host, may be NULL: 1 if the layer fell back, else 0
 *   err_host  host, may be NULL: the two errors of the split, as err above
 * Synchronous: it waits for `stream` to read the two errors back.
 */
sq_status sq_decompose_pack_auto(const float *W, int32_t N, int32_t K, int32_t trunk_percent,
                                 sq_packed_weight *out, void *scratch, size_t scratch_bytes,
                                 int32_t *fell_back, double *err_host, int32_t *dev_status,
                                 void *stream);

/*
 * Outlier calibration (m.lqnn.cn section 2.2: detect the outlier channels once,
 * cache their indices, look them up at run time).
 *   X        [T][K] f32 calibration activations, device
 *   k        number of channels to keep, 1 <= k <= K
 *   idx_out  [k] i32, device: the k channels with the largest max_t |X[t][j]|
 *            (ties: the lower channel first), sorted ascending.
 * K <= 40960.  Non-finite X counts as magnitude 0 and sets SQ_ERR_NONFINITE.
 */
sq_status sq_calibrate_outliers(const float *X, int32_t T, int32_t K, int32_t k,
                                int32_t *idx_out, int32_t *dev_status, void *stream);

/*
 * Per-token activation split (m.lqnn.cn section 2.2; dynamic per-token scale
 * of the visual guide's "动态量化" section).
 *   x          [M][K] f32 activations, device
 *   idx        [n_out] i32 outlier channels, strictly ascending in [0, K)
 *              (checked on the device: a violation sets SQ_ERR_INVALID_ARG)
 *   xq         [M][roundup(K,128)] i8 out: codes, 0 on outlier channels and pads
 *   sx         [M] f32 out: absmax over the non-outlier channels / 127
 *   x_out      [M][n_out] f32 out: the outlier channels, copied
 * 0 <= n_out <= 4096.  Non-finite x sets SQ_ERR_NONFINITE.
 */
sq_status sq_quantize_act(const float *x, int32_t M, int32_t K, const int32_t *idx,
                          int32_t n_out, int8_t *xq, float *sx, float *x_out,
                          int32_t *dev_status, uint32_t flags, void *stream);

/* Workspace bytes sq_linear() needs for this weight and token count on the
 * current device.  Layout: a partial-sum area whose size depends only on the
 * device (for rows split between warps), then one int32 arrival counter per
 * row (the last roundup(4*N, 256) bytes).  Zero-fill the workspace once
 * before its first use; every call leaves the counters zero again (the
 * partial sums are scratch).  One workspace may serve calls on different
 * weights, in stream order, if it is at least as large as each call needs. */
size_t sq_linear_workspace_bytes(const sq_packed_weight *w, int32_t M);

/*
 * Fused separated-quantization linear layer (m.lqnn.cn sections 2.3 and 3.3:
 * trunk by bit operations, residual by integer products, summed in one
 * kernel; the outlier channels of section 2.2 at full precision).
 *   w           packed weight (device arrays)
 *   xq, sx, x_out, idx, n_out   as written by sq_quantize_act
 *   M           tokens, M >= 1.  A weight in SQ_LAYOUT_TILES (or _SPARSE) runs on the
 *               tensor cores (INT8 MMAs for the residual codes and for the
 *               trunk bits expanded to 0/-1 bytes), in passes of up to 8
 *               tokens; SQ_LAYOUT_ROWS runs on the CUDA cores (dp4a), in
 *               passes of up to 4 tokens.  The results are the same.
 *   y           [M][N] f32 out
 *   workspace   device, ws_bytes >= sq_linear_workspace_bytes(w, M)
 * For every token t and row r:
 *   T  = sum_j m*(2b-1)*xq  = 2*sum_{m and b} xq - sum_m xq   (exact int32)
 *   R_g = sum_{j in g} q*xq                                     (exact int32)
 *   y  = sx*(alpha*T + sum_g s_g*R_g) + sum_i What[r][idx_i]*x_out[i]
 * with What = m*(+-alpha) + s_g*q the dequantized weight, in fp32.
 * flags: SQ_LAUNCH_PDL and/or SQ_TRUNK_ONLY (the residual terms dropped).
 */
sq_status sq_linear(const sq_packed_weight *w, const int8_t *xq, const float *sx,
                    const float *x_out, const int32_t *idx, int32_t n_out, int32_t M, float *y,
                    void *workspace, size_t ws_bytes, int32_t *dev_status, uint32_t flags,
                    void *stream);

/*
 * Same kernels as sq_linear, additionally writing the exact integer
 * accumulators for inspection:
 *   T_out [M][N] i32, R_out [M][N][ceil(K/G)] i32.
 * y is written as by sq_linear.  flags: 0.  Intended for tests; not on the
 * hot path.
 */
sq_status sq_linear_accumulators(const sq_packed_weight *w, const int8_t *xq, const float *sx,
                                 const float *x_out, const int32_t *idx, int32_t n_out,
                                 int32_t M, float *y, int32_t *T_out, int32_t *R_out,
                                 void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 uint32_t flags, void *stream);

/*
 * The activation split and the linear layer in one kernel (m.lqnn.cn
 * sections 2.2, 2.3 and 3.3: the split, the two products and their sum in a
 * single fused step).  For a weight in SQ_LAYOUT_TILES or SQ_LAYOUT_TILES_SPARSE.
 *   x           [M][K] f32 activations, device
 *   idx, n_out  outlier channels, strictly ascending in [0, K) (checked on
 *               the device: a violation sets SQ_ERR_INVALID_ARG)
 *   y           [M][N] f32 out
 *   workspace   at least sq_linear_workspace_bytes(w, M) bytes, 16-byte
 *               aligned, zero-filled before its first use (as for
 *               sq_linear); with sq_quantize_linear_workspace_bytes(w, M,
 *               n_out) bytes the staged route below may be taken
 * Every CTA forms the per-token scale, codes and outlier values of x in its
 * shared memory with the same arithmetic as sq_quantize_act, then runs the
 * decode of sq_linear: y is bit-identical to sq_quantize_act followed by
 * sq_linear.  Non-finite x sets SQ_ERR_NONFINITE.  Tokens are processed in
 * passes of up to 8 that fit the shared memory (roundup(K,128) +
 * 4*roundup(n_out,4) + 8192 bytes per token beside a fixed part); SQ_ERR_SHAPE
 * if not even one token fits (K above about 100000).
 * Staged route: when M > 1 and M*roundup(K,128) > 16384, or the tokens need
 * more fused passes than the decode kernel's passes of 8, and the workspace
 * is large enough, the call runs sq_quantize_act once into the workspace and
 * then sq_linear on its codes (two launches; y is the same bit for bit).
 * flags: SQ_LAUNCH_PDL (the kernel then reads x and writes y only after the
 * previous kernel completes; the packed weights and the index list are read
 * before, as for every SQ_LAUNCH_PDL launch) and/or SQ_TRUNK_ONLY.
 */
sq_status sq_quantize_linear(const sq_packed_weight *w, const float *x, int32_t M,
                             const int32_t *idx, int32_t n_out, float *y, void *workspace,
                             size_t ws_bytes, int32_t *dev_status, uint32_t flags, void *stream);

/*
 * Workspace bytes with which sq_quantize_linear may take its staged route:
 * sq_linear_workspace_bytes(w, M) rounded up to 256, then the activation
 * codes [M][roundup(K,128)] i8, the token scales [M] f32 and the outlier
 * values [M][n_out] f32, each 256-byte aligned.  Only the leading
 * sq_linear_workspace_bytes part must be zero-filled.  0 for an invalid
 * weight, M < 1, n_out out of range or no usable device.
 */
size_t sq_quantize_linear_workspace_bytes(const sq_packed_weight *w, int32_t M, int32_t n_out);

/*
 * Tokens that share one read of the weights in sq_linear's decode kernels for
 * this weight and flags (SQ_TRUNK_ONLY or 0): for the tiled layouts 16 where
 * the partial sums of 16 tokens fit in one CTA's shared memory beside its
 * tile ring (every shape up to K = 28672 with the dense symmetric residual),
 * else 8; for SQ_LAYOUT_ROWS 4 (below the prefill kernel's token count).  M
 * tokens take ceil(M / this) launches.  0 for an invalid weight or flags.
 */
int32_t sq_linear_tokens_per_pass(const sq_packed_weight *w, uint32_t flags);

/*
 * Tokens per launch of sq_quantize_linear's fused kernel for this weight and
 * outlier count (1..8; 0 if not even one token fits, or for an invalid
 * weight or a weight in SQ_LAYOUT_ROWS).
 */
int32_t sq_quantize_linear_tokens_per_pass(const sq_packed_weight *w, int32_t n_out);

/*
 * sq_linear without a caller workspace, for callers that cannot allocate
 * device memory at call time.  This entry point has no counterpart on the
 * pages: it only changes where the scratch lives.
 *   Scratch: one file-scope device array of SQ_LINEAR_NOALLOC_SCRATCH_BYTES
 *   (16 MiB) per device, inside this library.  Nothing is allocated.
 *   Limit: a call whose sq_linear_workspace_bytes(w, M) exceeds that size
 *   returns SQ_ERR_WORKSPACE before any device work (on a 148-SM B200: more
 *   than 4,118,528 rows).
 *   First call on each device: looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and zero-fills the
 *   array on `stream` before its launch, because the per-row arrival
 *   counters in it must start at zero.  Make that first call before any
 *   stream capture.  Every call leaves the counters zero again.
 *   Overlapping calls race: all calls on a device share the array, so two
 *   calls whose kernels may run at the same time (other streams, other host
 *   threads) give wrong results.  Order them on one stream or by events.
 *   The stream must belong to the current device (else SQ_ERR_INVALID_ARG):
 *   the array used is the current device's.
 * Arguments, flags and results are those of sq_linear.
 */
#define SQ_LINEAR_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
sq_status sq_linear_noalloc(const sq_packed_weight *w, const int8_t *xq, const float *sx,
                            const float *x_out, const int32_t *idx, int32_t n_out, int32_t M,
                            float *y, int32_t *dev_status, uint32_t flags, void *stream);

/* ---- NVFP4 prefill (format separation) ------------------------------------
 * The ISTA-DASLab news page on separated quantization, paragraphs 2-4:
 * prefill runs in the hardware's native quantized format, NVFP4, and decode
 * keeps its own low-bit weight-only format (the packed weights above).  A
 * layer then holds its weight twice: packed for decode and NVFP4 for
 * prefill.  The page names NVFP4 without defining it; the format here is the
 * one the B200 tensor cores read (tcgen05.mma kind::mxf4nvf4):
 *   element  E2M1, two per byte (the lower channel in the low nibble), sign
 *            in bit 3, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 in code order;
 *   block    16 consecutive channels share a UE4M3 scale s_b (no sign, 4
 *            exponent bits with bias 7, 3 mantissa bits, largest 448);
 *   tensor   a float second-level scale g = amax / (6 * 448): one per weight
 *            (per_row = 0), one per activation row, i.e. token (per_row = 1).
 * Quantization: s_b = nearest UE4M3 to amax_b / (6 g), q = nearest E2M1 to
 * x / (s_b g) saturating at +-6, ties to the even code, +0 for a zero
 * result; g = 0 or s_b = 0 gives zero codes.  Dequantized: e2m1(q) s_b g.
 *
 * Layout of one matrix [rows][K] (sq_nvfp4_view carves one allocation):
 *   codes   [rows_pad][code_stride] bytes, code_stride = roundup(K, 256) / 2,
 *           rows_pad = roundup(rows, 128); pads are 0
 *   scales  chunks of 512 bytes, chunk (rb, c) at byte 512 * (rb * sf_chunks
 *           + c), sf_chunks = roundup(K, 256) / 64: byte 16 i + 4 w + s of
 *           the chunk is the scale of row 128 rb + 32 w + i (i < 32, w < 4)
 *           and block 4 c + s (the tensor core's scale-factor layout); pads 0
 *   g       per_row: [rows_pad] floats (pads 0); else [2]: g, then a word the
 *           quantizer uses as scratch
 */
typedef struct {
  int32_t rows, K;
  int32_t per_row;      /* 0: one second-level scale (a weight); 1: one per row */
  int32_t rows_pad;     /* roundup(rows, 128) */
  int32_t code_stride;  /* bytes per row of codes: roundup(K, 256) / 2 */
  int32_t sf_chunks;    /* 64-channel scale chunks per 128-row block: roundup(K, 256) / 64 */
  uint8_t *codes;
  uint8_t *scales;
  float *g;
} sq_nvfp4_matrix;

/* Bytes of one NVFP4 matrix (all three arrays, 256-byte aligned pieces);
 * 0 for rows or K outside [1, 2^24] or [1, 2^20]. */
size_t sq_nvfp4_bytes(int32_t rows, int32_t K, int32_t per_row);
/* Carves `base` (sq_nvfp4_bytes of device memory, 256-byte aligned) into the
 * arrays of *out.  No device access. */
sq_status sq_nvfp4_view(void *base, int32_t rows, int32_t K, int32_t per_row,
                        sq_nvfp4_matrix *out);
/* Quantizes X [rows][K] (float, row-major) into *out (every array written,
 * pads included).  Per tensor (per_row = 0) it reduces X's absolute maximum
 * first (two kernels); per row it is one kernel.  Non-finite X sets
 * SQ_ERR_NONFINITE in dev_status (the codes are then unspecified). */
sq_status sq_nvfp4_quantize(const float *X, const sq_nvfp4_matrix *out, int32_t *dev_status,
                            void *stream);
/* y [x.rows][w.rows] (float, row-major) = sum_j What[n][j] * xhat[t][j] for
 * a per-tensor weight w (N = w.rows) and per-row activations x (M = x.rows
 * tokens) of the same K: one tcgen05 block-scaled GEMM launch, fp32
 * accumulation in tensor memory, y = g_w * g_x[t] * D.  A bounded wait that
 * runs out sets SQ_ERR_TIMEOUT in dev_status. */
sq_status sq_nvfp4_linear(const sq_nvfp4_matrix *w, const sq_nvfp4_matrix *x, float *y,
                          int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SQ_H */
