/*
 * fathom.h -- C ABI of the Fathom top-k key scan on NVIDIA B200 (sm_100a).
 *
 * Fathom ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded
 * KV Caches", arXiv 2609.17652) scores all n cached keys of a KV head for
 * its G query heads by reading only a query-chosen prefix of each key
 * channel's 4-bit code, then keeps the top k keys per query head.  The
 * passages cited below are sections of the yeyulingfeng.com article on the
 * paper; "方法一" is the bit-plane store, "方法二" the per-group reverse
 * water-filling, "先算一笔字节账" the byte accounting.
 *
 * Conventions for every entry point
 *   - Memory is owned by the caller.  The library never allocates, never
 *     frees and keeps no state between calls, except the per-thread last
 *     CUDA error code, one fault word per device (fathom_device_status) and
 *     the fixed scratch array of fathom_scan_topk_noalloc, both static
 *     device objects of the library.  Pointers marked DEVICE must be readable (or
 *     writable) by the current CUDA device: device memory, managed memory,
 *     or, where stated, page-locked host memory mapped into the device's
 *     address space.  Pointers marked HOST are ordinary host memory.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) on the current device.  Outputs are valid
 *     once the stream reaches the call.  The decode-step kernels (plan, scans,
 *     threshold, top-k, union) are launched with programmatic dependent
 *     launch: each waits for the previous kernel in the stream to complete
 *     before it reads anything, so ordering is that of plain launches (also
 *     under CUDA graph capture), while the next kernel's launch overlaps the
 *     current one's tail.
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and returns a negative status.
 *   - A "group" is one KV head of one layer (its G query heads share one
 *     plan, so each key byte is read once, 方法二 last paragraph).  Arrays
 *     indexed [H] run over the groups of one call.
 *   - Layout names list dimensions outermost first; all arrays are dense
 *     row-major unless a stride argument says otherwise.
 *   - Limits: 32 <= D <= 256 with D % 32 == 0; 1 <= G <= 8; 1 <= k <= 4096
 *     and G*k <= 16384 for top-k (k <= 1024 on the candidate path); n < 2^31.
 */
#ifndef FATHOM_H
#define FATHOM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* fathom_stream_t; /* same type as cudaStream_t */

/* Status codes. */
#define FATHOM_OK 0
#define FATHOM_ERR_INVALID_ARG (-1) /* null/unreadable pointer, size or range error */
#define FATHOM_ERR_UNSUPPORTED (-2) /* D, G, k or alignment outside the limits above */
#define FATHOM_ERR_CUDA (-3)        /* a CUDA call failed; see fathom_last_cuda_error() */
#define FATHOM_ERR_WORKSPACE (-4)   /* caller buffer smaller than the *_bytes() query */
#define FATHOM_ERR_TIMEOUT (-5)     /* a bounded device wait gave up; see fathom_device_status() */
#define FATHOM_ERR_OVERFLOW (-6)    /* candidate pass could not prove its top-k exact */
#define FATHOM_ERR_BOUNDS (-7)      /* debug build only: a device-side bounds check failed (the access was skipped) */

/* Key element types for fathom_pack. */
#define FATHOM_KEYS_F32 0
#define FATHOM_KEYS_BF16 1

/* Output modes of fathom_scan. */
#define FATHOM_SCAN_DENSE 0
#define FATHOM_SCAN_CANDIDATE 1 /* PREPARE then FILTER, in one call */
#define FATHOM_SCAN_PREPARE 2   /* threshold pass only */
#define FATHOM_SCAN_FILTER 3    /* main candidate pass only, after PREPARE */

/* Library version as 10000*major + 100*minor + patch. */
int fathom_version(void);

/* Static, human-readable text for a status code. */
const char* fathom_status_string(int status);

/* The cudaError_t value behind the calling thread's last FATHOM_ERR_CUDA
 * (0 if none). */
int fathom_last_cuda_error(void);

/* Words per plane row for n tokens: ceil(n/64) rounded up to a multiple of
 * 16, i.e. 128-byte rows.  Any nb_stride >= ceil(n/64) that is even is
 * accepted; this value is the recommended one. */
int64_t fathom_nb_stride(int64_t n);

/*
 * fathom_pack -- build the bit-plane index of H groups (方法一).
 *
 * For group h, channel j and 64-token block b (tokens 64b .. 64b+63 that
 * are < n):
 *   m = max |k| over the block's tokens, s = m rounded to fp16 (nearest,
 *   ties to even), and each key gets the 4-bit code
 *   c = clamp(floor(8 k / s) + 8, 0, 15)    (c = 8 when s is 0 or infinite),
 * i.e. 16 uniform cells of width s/8 over [-s, s]; code 8 is the cell
 * [0, s/8) and the top bit of c is the sign (1 for k >= 0).  Plane p
 * (p = 0 is the top bit, read first) of channel j holds bit (3-p) of the
 * 64 codes of block b in one 64-bit word, token 64b+i at bit i:
 *   planes[((h*D + j)*4 + p)*nb_stride + b],
 * so each plane row is contiguous along the sequence.  Bits of tokens >= n
 * are 0.  Storage: 4 x 8 B + 2 B per channel per 64 tokens = 68 B per token
 * per KV head at D = 128.
 *
 *   keys        DEVICE, key_dtype elements; token i of group h, channel j at
 *               keys[h*key_stride_h + i*key_stride_tok + j] (element units;
 *               channels contiguous).  Values should be finite with
 *               |k| < 65520 (fp16 range of the scale).
 *   key_dtype   FATHOM_KEYS_F32 or FATHOM_KEYS_BF16.
 *   H, n, D     groups, tokens, channels.  H == 0 or n == 0 is a no-op.
 *   planes      DEVICE out, uint64 [H][D][4][nb_stride], 8-byte aligned.
 *   scales      DEVICE out, fp16 bit patterns [H][D][nb_stride].
 *   nb_stride   words per plane row, >= ceil(n/64) and even.
 * Words/scales at block indices >= ceil(n/64) are not written.
 *
 * Appending during decode: new tokens land in the tail block, whose scale
 * (its maximum) can change, so the tail block is quantised again from its
 * raw keys.  Call fathom_pack on the keys from token 64*b0 onwards with
 * planes + b0 and scales + b0 (same nb_stride as the whole index): blocks
 * b0.. are rewritten, earlier blocks are untouched, and the result equals
 * packing all tokens at once.
 */
int fathom_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
                int64_t key_stride_h, int64_t key_stride_tok,
                uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                fathom_stream_t stream);

/*
 * fathom_pack_rotated -- the index of the keys' coordinates in an
 * orthonormal basis U (基座选择: for models without QK-norm the planes hold
 * each key in the KLT basis of the calibration keys, and the queries are
 * rotated the same way, q'_i = sum_d q_d U[d][i], so q'.y = q.k).  Equal to
 * fathom_pack of the rotated keys y [H][n][D], which are never written:
 *   y_i = sum_d k_d U[h][d][i], summed over d = 0, 1, ..., D-1 in that order
 *   from +0, every step one fp32 fused multiply-add (one rounding).
 * The order is part of the definition: the planes are bit-exact against any
 * evaluation of the same chain.
 *
 *   keys, key_dtype, H, n, D, key strides, planes, scales, nb_stride
 *               as for fathom_pack (keys finite; the rotated coordinates
 *               must stay below 65520 in magnitude).
 *   U           DEVICE, fp32 [H][D][D], contiguous: U[(h*D + d)*D + i] is
 *               component d of direction i (columns are the directions).
 * Cost: D fused multiply-adds per coordinate per token (FP32-pipe bound).
 * Appending works as for fathom_pack (rewrite from the tail block on).
 */
int fathom_pack_rotated(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
                        int64_t key_stride_h, int64_t key_stride_tok, const float* U,
                        uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                        fathom_stream_t stream);

/*
 * fathom_calibrate_workspace_bytes -- scratch fathom_calibrate needs (HOST
 * call); 0 for unsupported sizes.
 */
size_t fathom_calibrate_workspace_bytes(int64_t H, int D, int with_cov);

/*
 * fathom_calibrate -- per-group key statistics over the first n keys: the
 * channel variance sigma^2 that fathom_plan takes (方法二: measured once on
 * calibration keys), and optionally the mean and the covariance from which
 * a caller builds a rotated basis (实验 section: statistics from the
 * session's own prefill keys, one covariance per KV head).
 *
 *   mean_j  = (1/n) sum_i k_ij
 *   sigma2_j = (1/n) sum_i (k_ij - mean_j)^2            (population variance)
 *   cov_ab  = (1/n) sum_i (k_ia - mean_a)(k_ib - mean_b)
 *
 * Sums run in double precision over k - k_0 (the group's first key) and are
 * rounded once to fp32; the double atomics that combine chunks make the
 * last fp64 bits depend on timing, so an output can differ between runs
 * only where its fp64 value lies next to an fp32 rounding boundary.
 *
 *   keys        DEVICE, [H][n][D] as for fathom_pack (fp32 or bf16, strides in
 *               elements); not read when n == 0.
 *   mean        DEVICE out (may be NULL), fp32 [H][D].
 *   sigma2      DEVICE out, fp32 [H][D].
 *   cov         DEVICE out (may be NULL), fp32 [H][D][D].
 *   workspace, ws_bytes  DEVICE scratch of at least
 *               fathom_calibrate_workspace_bytes(H, D, cov != NULL) bytes,
 *               256-byte aligned (FATHOM_ERR_WORKSPACE if smaller).
 * n == 0 gives zeros.  D as for fathom_pack; H <= 65535.
 */
int fathom_calibrate(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
                     int64_t key_stride_h, int64_t key_stride_tok, float* mean, float* sigma2,
                     float* cov, void* workspace, size_t ws_bytes, fathom_stream_t stream);

/*
 * fathom_plan -- per-group reverse water-filling (方法二).
 *
 * Channel importance, in single precision with round-to-nearest and in this
 * exact order (no fused multiply-add):
 *   w_j = sigma2_j * ((((q_{0,j}^2 + q_{1,j}^2) + q_{2,j}^2) + ...) + q_{G-1,j}^2).
 * Reading t planes leaves error variance proportional to 4^-t, so the
 * (t+1)-th plane of channel j is worth the item w_j * 4^-t (t = 0..3).
 * The water level theta* is the smallest theta >= 0 for which
 *   sum_j t_j(theta) <= B,  t_j(theta) = #{t in 0..3 : w_j 4^-t > theta},
 * i.e. the (B+1)-th largest positive item, or 0 when at most B items are
 * positive; depth_j = t_j(theta*).  Ties at theta* are all left unread, so
 * sum_j depth_j can be below B.  Items are compared exactly.  The search is
 * a bisection on an integer key that is monotone in log theta and ends
 * exactly (at most 32 halvings).
 *
 *   sigma2       DEVICE, fp32 [H][D], per-channel key variance (calibration).
 *   q            DEVICE, fp32 [H][G][D], the group's query heads.
 *   budget_bits  DEVICE, int32 [H], plane bits per token per group (B); or
 *                NULL to use budget_flat for every group.  Values are
 *                clamped to [0, 4D].
 *   budget_flat  used when budget_bits is NULL; must be in [0, 4D].
 *   depth        DEVICE out, uint8 [H][D], t_j in 0..4.
 *   active       DEVICE out, uint16 [H][D]: the channels with t_j > 0 in
 *                ascending j, entry = j | (t_j << 8); entries past n_active
 *                are 0.
 *   n_active     DEVICE out, int32 [H].
 *   theta        DEVICE out (may be NULL), fp32 [H]: theta* rounded to fp32
 *                (informational; depths are decided exactly).
 */
int fathom_plan(const float* sigma2, const float* q, int64_t H, int G, int D,
                const int32_t* budget_bits, int32_t budget_flat,
                uint8_t* depth, uint16_t* active, int32_t* n_active, float* theta,
                fathom_stream_t stream);

/*
 * fathom_layer_budgets_workspace_bytes -- scratch fathom_layer_budgets needs
 * (HOST call); 0 for unsupported sizes.
 */
size_t fathom_layer_budgets_workspace_bytes(int64_t H, int D);

/*
 * fathom_layer_budgets -- per-layer plane-bit budgets from calibration
 * queries (方法二, per-layer plan paragraph: layers differ in how sharp
 * their scores are, and a greedy pass on calibration data can give each its
 * own budget; the pages' default stays the flat budget).  The groups of
 * layer l are h = l*P .. l*P + P - 1, P = H / layers, and all get B_l.
 * With w_j the plan's importance (same fp32 order) and v_h,(b) the b-th
 * largest item w_j 4^-t of group h, one more bit for layer l lowers its
 * error relative to its unread error sum_h sum_j w_hj by
 *   g_l(b) = 0.75 * sum_h v_h,(b) / sum_h sum_j w_hj.
 * The greedy gives total_bits (capped at layers * 4D) one bit at a time to
 * the layer with the largest next gain, ties to the lower layer, at most
 * 4D per layer; sums run in double in a fixed order, so the result is
 * defined bit for bit.  Pass budget_bits to fathom_plan.
 *
 *   sigma2, q   DEVICE, as for fathom_plan (q: calibration queries).
 *   layers      1..1024, dividing H.
 *   total_bits  the budget of all layers together (e.g. layers * 48).
 *   budget_bits DEVICE out, int32 [H].
 *   workspace, ws_bytes  DEVICE scratch of at least
 *               fathom_layer_budgets_workspace_bytes(H, D) bytes, 256-byte
 *               aligned.
 */
int fathom_layer_budgets(const float* sigma2, const float* q, int64_t H, int G, int D, int layers,
                         int64_t total_bits, int32_t* budget_bits, void* workspace, size_t ws_bytes,
                         fathom_stream_t stream);

/*
 * fathom_plan_fixed -- a fixed-depth comparator plan: the r channels with
 * the largest a_j = |q_{0,j}| + |q_{1,j}| + ... + |q_{G-1,j}| (single
 * precision, that order; ties to the lower j) read at `bits` planes, the
 * others at 0.  The group's heads share the channel set so the K bytes are
 * read once.  The comparators of the pages (先算一笔字节账 and 固定深度的浪费在哪):
 *   r = 32, bits = 4: the 136-bit scan (32 coordinates x 4 bits + scales);
 *   r = 16, bits = 4: SparQ's 68-bit read;
 *   r = D,  bits = 2: the thumbnail scan (2 bits of every channel).
 * Outputs as fathom_plan.  0 <= r <= D, 1 <= bits <= 4.
 */
int fathom_plan_fixed(const float* q, int64_t H, int G, int D, int r, int bits,
                      uint8_t* depth, uint16_t* active, int32_t* n_active,
                      fathom_stream_t stream);

/*
 * fathom_scan_cand_bytes -- size of the candidate buffer fathom_scan needs
 * in FATHOM_SCAN_CANDIDATE mode for these sizes (HOST call, no GPU work).
 */
size_t fathom_scan_cand_bytes(int64_t H, int G, int64_t n, int k);

/*
 * fathom_scan -- variable-depth scores (方法一 prefix reads, 方法二 plan).
 *
 * For group h, query head g and token i < n:
 *   score_{g,i} = sum_{(j,t) in active[h]} q_{g,j} * khat_{i,j},
 *   khat = s_{b,j} * (2 c_t - 2^t + 1) / 2^t,   c_t = the first t planes'
 * bits of the key's code (the t-bit mid-rise quantiser on [-s, s]), b = i/64.
 * Only the first t plane rows of each active channel and its scale row are
 * read; every plane word is read once for all G heads.  Arithmetic is fp32
 * (coefficients q * s * 2^-t rounded once, one fused multiply-add per
 * term); the result is within 1e-5 * sum_j |q_{g,j} khat_{i,j}| of exact
 * for D <= 128.  No 1/sqrt(D) factor is applied (it does not change ranks).
 *
 *   planes, scales  DEVICE (or mapped page-locked host memory), as written
 *                   by fathom_pack with the same nb_stride.  Both must be
 *                   16-byte aligned and nb_stride a multiple of 8 (as
 *                   fathom_nb_stride() gives); FATHOM_ERR_UNSUPPORTED
 *                   otherwise.
 *   active, n_active  DEVICE, from fathom_plan / fathom_plan_fixed.
 *   q               DEVICE, fp32 [H][G][D].
 *   mode            FATHOM_SCAN_DENSE: write scores.
 *                   FATHOM_SCAN_CANDIDATE: write into cand only the keys
 *                   whose score reaches a per-head threshold tau taken
 *                   from a 1-in-S tile sample of the same scores (S chosen
 *                   from n and k; tau = -inf when n is small), so that
 *                   fathom_topk can select from them.  The threshold is a
 *                   filter only: fathom_topk checks that at least k keys
 *                   passed and none were dropped, which proves the top-k
 *                   exact, and flags the group otherwise.
 *                   FATHOM_SCAN_PREPARE: only the threshold part (sample
 *                   pass, tau per head, counters reset to 0).
 *                   FATHOM_SCAN_FILTER: only the main pass, appending to a
 *                   cand buffer that a PREPARE call with the same H, G, n, k
 *                   readied earlier on the stream.  CANDIDATE is PREPARE
 *                   followed by FILTER; the split lets a caller time or
 *                   overlap the two.
 *   scores          DEVICE out, fp32 [H][G][n] (DENSE; ignored otherwise).
 *   cand, cand_bytes  DEVICE scratch/out of at least
 *                   fathom_scan_cand_bytes(H, G, n, k) bytes (all modes but
 *                   DENSE, which ignores it), 16-byte aligned.
 *   k               winners per query head that will be asked of
 *                   fathom_topk (sizes the candidate pass).
 *
 * The kernel hands plane rows from a loader warp to the compute warps
 * through a shared-memory ring whose waits are bounded.  A wait that gives
 * up (which a correct launch never does) sets the device fault word and
 * the launch's outputs are void: fathom_topk then reports
 * FATHOM_ERR_TIMEOUT, and fathom_device_status() returns it.
 */
int fathom_scan(const uint64_t* planes, const uint16_t* scales, int64_t H, int D,
                int64_t n, int64_t nb_stride, const uint16_t* active,
                const int32_t* n_active, const float* q, int G, int mode,
                float* scores, void* cand, size_t cand_bytes, int k,
                fathom_stream_t stream);

/*
 * fathom_nibbles_from_planes -- the same 4-bit codes stored whole: for each
 * (group, channel, block) four 64-bit words, word w holding tokens
 * 16w .. 16w+15 of the block, token 16w + e in bits 4e .. 4e+3.  Layout
 * [H][D][4][nb_stride], like the planes (a row (h, j, w) is contiguous along
 * the blocks), and the scales are the planes' own.  This is the store a
 * fixed-depth scan reads (先算一笔字节账: 32 coordinates at 4 bits plus a
 * block scale), kept as a comparator: its bytes per read coordinate equal
 * the planes' at depth 4, so the two scans differ only in decoding.
 *
 *   planes      DEVICE, as written by fathom_pack.
 *   nibbles     DEVICE out, uint64 [H][D][4][nb_stride].
 */
int fathom_nibbles_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n, int64_t nb_stride,
                               uint64_t* nibbles, fathom_stream_t stream);

/*
 * fathom_scan_nibbles -- fathom_scan over the nibble store: every active
 * channel is read whole (4 bits; the plan's depths are ignored), so it
 * computes the scores of fathom_scan with every active depth at 4, bit for
 * bit.  Arguments, modes, outputs and errors are fathom_scan's, with
 * `nibbles` in place of `planes`.
 */
int fathom_scan_nibbles(const uint64_t* nibbles, const uint16_t* scales, int64_t H, int D,
                        int64_t n, int64_t nb_stride, const uint16_t* active,
                        const int32_t* n_active, const float* q, int G, int mode,
                        float* scores, void* cand, size_t cand_bytes, int k,
                        fathom_stream_t stream);

/*
 * fathom_nibbles_tm_from_planes -- the same 4-bit codes stored TOKEN-MAJOR,
 * as a serving stack keeps a 4-bit K cache: token i of group h owns one row
 * of D/2 bytes, byte c holding channel 2c in its low nibble and channel
 * 2c + 1 in its high nibble:
 *   store[(h * 64 * nb_stride + i) * (D/2) + c],
 * rows for tokens 0 .. 64*ceil(n/64) - 1 written (tokens past n hold code
 * 0).  Scales stay the planes' own.  A scan of r chosen channels moves whole
 * rows: D/2 bytes per token per KV head (64 B at D = 128) whatever r is,
 * against r/2 bytes in the channel-major stores (先算一笔字节账: the
 * fixed-depth scans' 4-bit coordinates).
 *
 *   planes      DEVICE, as written by fathom_pack.
 *   store       DEVICE out, uint8 [H][64*nb_stride][D/2], 16-byte aligned.
 */
int fathom_nibbles_tm_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n,
                                  int64_t nb_stride, uint8_t* store, fathom_stream_t stream);

/*
 * fathom_scan_nibbles_tm -- fathom_scan_nibbles over the token-major store:
 * every active channel read at 4 bits, value (c - 7.5) s/8 with the
 * channel's block scale.  Arguments, modes, outputs and errors are
 * fathom_scan's, with `store` in place of `planes` (the candidate buffer
 * and fathom_topk are shared).  Scores agree with fathom_scan_nibbles to
 * fp32 rounding (the sums run in another order).
 */
int fathom_scan_nibbles_tm(const uint8_t* store, const uint16_t* scales, int64_t H, int D,
                           int64_t n, int64_t nb_stride, const uint16_t* active,
                           const int32_t* n_active, const float* q, int G, int mode,
                           float* scores, void* cand, size_t cand_bytes, int k,
                           fathom_stream_t stream);

/*
 * fathom_topk_workspace_bytes -- scratch fathom_topk needs (HOST call).
 */
size_t fathom_topk_workspace_bytes(int64_t H, int G, int64_t n, int k);

/*
 * fathom_topk -- per query head, the k keys with the largest scores, ties
 * broken towards the lower token index, listed by (score descending, index
 * ascending); then per group the ascending, de-duplicated union of its G
 * winner lists (at most G*k keys; 先算一笔字节账, top-k bullet).
 *
 * Scores are ordered as fp32 values (-0 equals +0).  Exactly one of
 * scores / cand is non-NULL:
 *   scores     DEVICE, fp32 [H][G][n] from a DENSE scan.
 *   cand       DEVICE, the candidate buffer of a CANDIDATE scan with the
 *              same H, G, n, k.  The call also uses one counter word of
 *              each group's header in it (left as it found it), so two
 *              fathom_topk calls on one candidate buffer must not overlap
 *              on the GPU.
 *   idx        DEVICE out, int32 [H][G][k].
 *   union_idx  DEVICE out, int32 [H][G*k], ascending, -1 padded.
 *   union_count DEVICE out, int32 [H]: size of each union, or
 *              FATHOM_ERR_OVERFLOW for a group whose candidate pass kept
 *              fewer than k or more than its capacity of keys; such a
 *              group's idx and union_idx are unspecified and the caller
 *              reruns it with a DENSE scan; FATHOM_ERR_TIMEOUT for every
 *              group while the device fault word is set (a scan's bounded
 *              wait gave up: nothing of that step is valid), or
 *              FATHOM_ERR_BOUNDS in a debug build whose bounds check failed.
 *   workspace, ws_bytes  DEVICE scratch of fathom_topk_workspace_bytes()
 *              bytes (may be NULL when that is 0).
 */
int fathom_topk(const float* scores, const void* cand, int64_t H, int G, int64_t n, int k,
                int32_t* idx, int32_t* union_idx, int32_t* union_count,
                void* workspace, size_t ws_bytes, fathom_stream_t stream);

/*
 * fathom_dequant_rows -- rebuild whole key rows from the index: for group h
 * and list entry r < row_count[h] (all M entries when row_count is NULL),
 * token i = rows[h*M + r] and every channel j,
 *   out[(h*M + r)*D + j] = s_{i/64,j} * (2 c_t - 2^t + 1) / 2^t,  t = bits,
 * the t-plane prefix value of the stored code (t = 4: the full 4-bit key).
 * This is how the keys of a KV head's winners can be served from the
 * channel-major planes themselves (边界, storage-overhead paragraph: the
 * pages leave this path unbuilt and note a single token is costly to gather
 * from the channel-major layout).  Values are exact in fp32.  Entries with
 * i outside [0, n) and rows past row_count give 0.
 *
 *   planes, scales  as for fathom_scan (device or mapped host memory).
 *   rows            DEVICE, int32 [H][M] token indices (e.g. the union of
 *                   fathom_topk, ascending, which keeps the reads local).
 *   row_count       DEVICE (may be NULL), int32 [H]; negative counts read as 0.
 *   bits            1..4.
 *   out             DEVICE out, fp32 [H][M][D].
 */
int fathom_dequant_rows(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                        int64_t nb_stride, const int32_t* rows, int64_t M, const int32_t* row_count,
                        int bits, float* out, fathom_stream_t stream);

/*
 * fathom_union_attention_workspace_bytes -- scratch fathom_union_attention
 * needs (HOST call); 0 for unsupported sizes.
 */
size_t fathom_union_attention_workspace_bytes(int64_t H, int G, int D, int64_t M);

/*
 * fathom_union_attention -- the step after the scan: each query head's
 * softmax attention over the KV rows of its group's union of winners (先算
 * 一笔字节账, top-k bullet: a step fetches the union of the G heads'
 * winner rows, at most G*k per KV head).  For group h, head g and the rows
 * i = union_idx[h*M + r], r < union_count[h]:
 *   s_i = scale * q_g . K_i,   out_g = sum_i softmax(s)_i V_i.
 * fp32 arithmetic (expf); rows are taken in chunks of 256 and the chunks
 * combined by their maxima (split over the union).  A union_count <= 0
 * (none, or an error status from fathom_topk) gives a zero output; an
 * index outside [0, n) is skipped.
 *
 *   k_cache, v_cache  DEVICE, [H][n][D] fp32 or bf16 (kv_dtype), the
 *               session's full-precision cache, strides in elements.
 *   q           DEVICE, fp32 [H][G][D].
 *   union_idx, union_count  DEVICE, as fathom_topk writes them (M = G*k).
 *   scale       usually 1/sqrt(D).
 *   out         DEVICE out, fp32 [H][G][D].
 *   workspace, ws_bytes  DEVICE scratch of at least
 *               fathom_union_attention_workspace_bytes(H, G, D, M) bytes,
 *               256-byte aligned.
 * 1 <= M <= 65536; D, G as for fathom_plan; H <= 65535.
 */
int fathom_union_attention(const void* k_cache, const void* v_cache, int kv_dtype, int64_t H, int64_t n,
                           int D, int64_t kv_stride_h, int64_t kv_stride_tok, const float* q, int G,
                           const int32_t* union_idx, const int32_t* union_count, int64_t M, float scale,
                           float* out, void* workspace, size_t ws_bytes, fathom_stream_t stream);

/*
 * fathom_scan_topk_noalloc -- fathom_scan in CANDIDATE mode followed by
 * fathom_topk, for callers that cannot allocate device memory.  (The paper
 * has no counterpart: this is a deployment convenience of this library.)
 *
 * Some callers cannot hand the scan a scratch buffer: an operator plugged
 * into another inference runtime that has already reserved the free device
 * memory for its KV-cache pool and gives the operator no allocator, or a
 * decode loop that must not call cudaMalloc because it synchronises the
 * device.  This call keeps the candidate buffer in an array that the
 * library itself owns in device memory, of FATHOM_NOALLOC_SCRATCH_BYTES;
 * every device that loads the library holds that much until the process
 * exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 *
 * Arguments and results are those of fathom_scan (without mode, scores,
 * cand, cand_bytes) and of fathom_topk (without scores, cand, workspace):
 * union_count[h] == FATHOM_ERR_OVERFLOW still marks a group to rerun densely.
 * Sizes whose candidate buffer, fathom_scan_cand_bytes(H, G, n, k), exceeds
 * FATHOM_NOALLOC_SCRATCH_BYTES are rejected with FATHOM_ERR_WORKSPACE
 * before anything is launched (one layer of 8 KV heads with G = 4, k = 512
 * fits at n = 1M; a whole 288-group step does not -- call it per layer).
 *
 * The first call on a device looks up the array's device address (a
 * one-time cudaGetSymbolAddress with that device current); make that first
 * call before any stream capture.  All calls share the one array, and each
 * call's threshold pass resets the counters it uses, so leftover contents
 * never leak into a result; but calls whose work overlaps on the GPU (two
 * streams, or two threads on one device) race on the array and must be
 * serialised by the caller.
 */
#define FATHOM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

int fathom_scan_topk_noalloc(const uint64_t* planes, const uint16_t* scales, int64_t H, int D,
                             int64_t n, int64_t nb_stride, const uint16_t* active,
                             const int32_t* n_active, const float* q, int G, int k,
                             int32_t* idx, int32_t* union_idx, int32_t* union_count,
                             fathom_stream_t stream);

/*
 * fathom_device_status -- FATHOM_ERR_TIMEOUT if a kernel of this library on
 * the current device has given up a bounded wait since the word was last
 * cleared; else FATHOM_ERR_BOUNDS if, in a build with device-side bounds
 * checks (FATHOM_DEBUG_BOUNDS), a check failed and its access was skipped;
 * else FATHOM_OK (or FATHOM_ERR_CUDA).  (The paper has no counterpart: this
 * is the library's own failure report.)
 *
 * Reads the device's fault word in stream order and synchronises `stream`;
 * with clear != 0 a set word is reset to 0 afterwards.  The word is one per
 * device and process, so a fault seen here may come from work on another
 * stream.  The first call on a device looks the word's address up (a
 * one-time cudaGetSymbolAddress), as the first scan on that device does.
 */
int fathom_device_status(int clear, fathom_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FATHOM_H */
