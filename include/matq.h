/*
 * matq.h -- C ABI of libmatq: sliced r-bit ("Matryoshka") linear layers on B200 (sm_100a).
 *
 * A weight matrix W [N, K] (torch.nn.Linear layout: N outputs, K inputs, K contiguous)
 * is stored as ONE set of unsigned 8-bit parent codes q in [0, 255] with one fp16 scale s
 * and one unsigned 8-bit zero point z per group of `group` consecutive inputs of a row.
 * The scale and zero point are shared by every width ("Matryoshka Quantization | Summary",
 * §3.1 MinMax quantizer; MatQuant rebuttal page, S.P. MatQuant item 2; "MatGPTQ: Efficient
 * and Accurate Inference over Nested Quantized Models" §1, single shared-scale format).
 *
 * A width-r model, r in {2, 3, 4, 6, 8}, uses only the r most significant bits of every
 * code (true-prefix slicing, MatGPTQ App. A.1):
 *
 *     p       = q >> (8 - r)                         (the prefix, 0 <= p < 2^r)
 *     q_hat   = p * 2^(8-r) + delta_r,   delta_r = (2^(8-r) - 1) / 2
 *     W_hat   = s * (q_hat - z)
 *     y[m, n] = sum_k x[m, k] * W_hat[n, k]         (MatGPTQ §4: Y = X W_D)
 *
 * delta_r centres the value in its cell (App. A.1) and is folded into the zero point
 * inside the kernels; a width-r call reads exactly r bits per weight (MatGPTQ §4).
 *
 * Conventions for every entry point
 *   - All data pointers are caller-owned DEVICE memory unless stated; the library never
 *     allocates, frees or keeps pointers between calls.
 *   - `stream` is a cudaStream_t (0 = legacy default stream).  Every call is asynchronous
 *     on that stream; a returned MATQ_OK means "validated and launched", not "finished".
 *   - Every call returns an int status: MATQ_OK (0) or a negative MATQ_E* code.  Argument
 *     errors are caught on the host before any launch and leave every buffer untouched.
 *     A launch failure returns MATQ_ECUDA; matq_last_cuda_error() gives the cudaError_t.
 *   - Shapes: N >= 1; K a positive multiple of 256 (matq_choose_codes: of group); M >= 1.
 *     group in {64, 128}.
 *   - Alignment: every device pointer must be 16-byte aligned.
 *   - Thread safety: calls on different streams may run concurrently (with separate
 *     workspaces); the only state is a thread-local "last CUDA error" and per-device caches of
 *     launch settings, except matq_linear_noalloc, whose calls on one device share a
 *     library-owned scratch array and must be ordered (see its contract).
 *
 * Packed plane layout ("MATQ-PL1"; written by matq_pack, read by every other call)
 *   The 8 code bits are split into five planes, most significant first:
 *       plane 0: bits 7..6 (2 bits/weight)   plane 1: bit 5      plane 2: bit 4
 *       plane 3: bits 3..2 (2 bits/weight)   plane 4: bits 1..0
 *   Width r reads planes 0..P(r)-1 with P(2)=1, P(3)=2, P(4)=3, P(6)=4, P(8)=5; the bits of
 *   those planes sum to r.  (The split into {1-2, 3, 4, 5-6, 7-8} MSB planes follows
 *   MatGPTQ §4; the order of bits inside a plane is this library's own.)
 *   Planes are stored back to back, plane 0 first, so the first matq_packed_bytes(N, K, r)
 *   bytes of any pack with r_keep >= r are themselves a valid width-r pack ("mode A":
 *   keep only the r-bit prefix resident; "mode B": keep all 8 bits and pass r per call).
 *   Inside a plane of b bits/weight (b = 1 or 2) the matrix is cut into row tiles of 16 rows
 *   (RT = ceil(N/16); rows >= N are packed as code 0) and K-chunks of 256 inputs
 *   (KC = K/256).  Tile (rt, kc) occupies b*512 bytes at byte offset (rt*KC + kc)*b*512.
 *   Inside a tile, the 4096 weights are dealt to 32 "lanes" (lane = 4*gid + tg, gid in 0..7,
 *   tg in 0..3), 128 weights each, in the operand order of a 16x16 fp16 MMA tile:
 *     block w in 0..7 covers inputs 32w..32w+31 of the chunk; in block w a lane holds 16
 *     fields f = 0..15 with u = f & 7, hi = f >> 3, j = u >> 2, rho = u & 3 and
 *         row = 16*rt + gid + 8*(rho & 1)
 *         k   = 256*kc + 32*w + 16*j + 2*tg + 8*(rho >> 1) + hi.
 *   2-bit planes: lane word w (w = 0..7) holds field f of block w in bits [2f, 2f+2); the
 *     tile is two 512-byte halves: words 0..3 of all lanes (lane-major, 16 bytes a lane),
 *     then words 4..7.
 *   1-bit planes: lane word v (v = 0..3) holds blocks 2v + a (a = 0, 1), field f of block
 *     2v + a at bit 4*(f >> 1) + 2*a + (f & 1); the tile is 32 lanes x 16 bytes.
 *   So a warp streams each plane with 16-byte-per-lane coalesced loads, and a lane's words
 *   turn into MMA operand registers with a few shifts and masks.
 */
#ifndef MATQ_H
#define MATQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------------ */
#define MATQ_OK             0
#define MATQ_EINVAL_R      -1   /* r not in {2,3,4,6,8}, or r > r_keep is MATQ_ETRUNC     */
#define MATQ_EINVAL_SHAPE  -2   /* N < 1, M < 1, K < 256 or K % 256 != 0, overflow          */
#define MATQ_EINVAL_GROUP  -3   /* group not in {64, 128}                                   */
#define MATQ_EALIGN        -4   /* a device pointer is not 16-byte aligned                  */
#define MATQ_ENULL         -5   /* a required pointer is NULL                               */
#define MATQ_ETRUNC        -6   /* the pack holds fewer planes than width r needs           */
#define MATQ_ECUDA         -7   /* a CUDA call or launch failed: see matq_last_cuda_error   */
#define MATQ_ESIZE         -8   /* a caller buffer (planes, workspace) is too small          */
#define MATQ_EDTYPE        -9   /* unknown output mode                                      */
#define MATQ_EDEVICE      -10   /* current device is not sm_100 (B200 class)               */
#define MATQ_ESCRATCH     -11   /* sizes exceed matq_linear_noalloc's fixed scratch        */
#define MATQ_EINVAL_ARG   -12   /* a lambda < 0 or not finite, or an unknown slicing mode  */

/* ---- output modes of matq_linear ----------------------------------------------------- */
#define MATQ_OUT_BF16       0   /* y [M, N] bf16 = x . W_hat^T                             */
#define MATQ_OUT_F32        1   /* y [M, N] fp32 = x . W_hat^T                             */
#define MATQ_OUT_F32_ACCUM  2   /* y [M, N] fp32 += x . W_hat^T (fused residual add)       */
#define MATQ_OUT_SILU_GATED 3   /* y [M, N/2] bf16 = silu(gate) * up, rows paired (below)  */

/* Library version (major*10000 + minor*100 + patch). */
int matq_version(void);

/* Human-readable text of a status code (static storage, never NULL). */
const char* matq_strerror(int status);

/* cudaError_t of the last failing CUDA call made by this thread (0 if none). */
int matq_last_cuda_error(void);

/* ---- layout queries (host only, no CUDA call) ---------------------------------------- */

/* Number of planes width r reads: 1, 2, 3, 4, 5 for r = 2, 3, 4, 6, 8; 0 if r is invalid. */
int matq_plane_count(int r);

/* Bytes of planes needed to serve every width <= r_keep:
 *     ceil(N/16) * 16 * K * r_keep / 8     (exactly r_keep bits per weight when 16 | N).
 * Returns 0 on invalid arguments (N < 1, K % 256 != 0, r_keep not a valid width). */
size_t matq_packed_bytes(int N, int K, int r_keep);

/* ---- one-time pack (§ "efficient packing", MatGPTQ §1 contribution 3 and §4) ---------- */

/* Repack parent codes into the MATQ-PL1 plane layout, keeping the planes of widths
 * <= r_keep.
 *   codes        [N, K] uint8, row-major, device.  Read only.
 *   planes       device buffer of at least matq_packed_bytes(N, K, r_keep) bytes; written.
 *   planes_bytes capacity of `planes` (MATQ_ESIZE if too small).
 * Every code byte is read once and every plane bit written once. */
int matq_pack(const uint8_t* codes, int N, int K, int r_keep,
              void* planes, size_t planes_bytes, void* stream);

/* Recover the width-r prefixes p = q >> (8 - r) from a pack (verification and export).
 *   planes     pack written with r_keep >= r (MATQ_ETRUNC otherwise).
 *   prefix_out [N, K] uint8, row-major, device; written. */
int matq_slice(const void* planes, int N, int K, int r_keep, int r,
               uint8_t* prefix_out, void* stream);

/* Deployment mode A: copy the width-r prefix of a pack (its first matq_packed_bytes(N,K,r)
 * bytes) into `planes_r`, which then is a width-r pack (r_keep = r) on its own.
 *   bytes  capacity of planes_r (MATQ_ESIZE if < matq_packed_bytes(N, K, r)). */
int matq_slice_copy(const void* planes, int N, int K, int r_keep, int r,
                    void* planes_r, size_t bytes, void* stream);

/* ---- the sliced linear layer ----------------------------------------------------------- */

/* Workspace bytes for matq_linear at these sizes (a multiple of 256): with this much every path
 * runs in its fastest form.  A prefill call (M > 16) whose matrix leaves most SMs without a
 * (row block, token tile) splits K and adds partial sums in the workspace; given less room
 * than that (but at least the header, 262,400 bytes, plus M*K*2 and M*4 bytes, each rounded up
 * to 256) it runs unsplit.  Decode calls need exactly this size.
 * A workspace starts with a fixed header (device status words and the ticket counters with
 * which the CTAs sharing a split row group elect the one that adds their partial sums; no CTA
 * waits for another).  The header must be zero-filled once before the first call
 * (matq_workspace_init, or any zero fill); every call leaves the counters zero again, so a
 * workspace is reused without re-initialisation.  Calls that share a workspace must be
 * ordered on the device (one stream, or synchronised streams).  A workspace sized for
 * (M_max, K_max, N) serves every call with M <= M_max and K <= K_max on either path
 * (a decode-sized one serves prefill only for M <= 16). */
size_t matq_linear_workspace(int M, int K, int N, int group);

/* Zero the workspace header (asynchronous on `stream`).  ws_bytes: capacity of workspace. */
int matq_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Synchronously read the device status left in the workspace header: 0 if every earlier call
 * completed normally; otherwise the OR of the codes of device-side waits that ran out (each
 * bounded wait gives up after about a second, records its code and lets the kernel return, so
 * the context stays usable).  The outputs of a call that recorded a code are undefined, and a
 * non-zero status requires matq_workspace_init before the workspace is used again. */
int matq_workspace_status(const void* workspace, int* status_out);

/* Status code recorded by matq_selftest_timeout. */
#define MATQ_STATUS_SELFTEST 0x100
/* Status code of a decode-path call (M <= 16) that met an activation with |x| >= 65536: the
 * decode path multiplies in fp16, which has no such value; that call's y is undefined. */
#define MATQ_STATUS_XRANGE 0x200

/* Failure-detection self-test (asynchronous on `stream`): launches one warp that waits, with the
 * same bounded wait every libmatq kernel uses, on a shared-memory barrier that nothing ever
 * completes.  After about a second the wait gives up, ORs MATQ_STATUS_SELFTEST into the decode
 * status word of `workspace` and the kernel returns; matq_workspace_status then reports it.
 * No GPU fault, trap or hang is involved. */
int matq_selftest_timeout(void* workspace, size_t ws_bytes, void* stream);

/* y = x . W_hat_r^T for a width-r slice of a pack.
 *   x        [M, K] bf16, row-major, device.  Read only.
 *   planes   pack with r_keep >= r.  Read only; exactly the planes of width r are read.
 *   scales   [N, K/group] fp16 (raw bits), row-major.  zeros [N, K/group] uint8.
 *   y        [M, N] row-major, dtype by y_mode (MATQ_OUT_*).  MATQ_OUT_SILU_GATED: N even and
 *            the weight rows interleave the gate and up projections of an FFN (row 2i: gate
 *            row i, row 2i + 1: up row i); y is [M, N/2] bf16 with y[m, i] =
 *            bf16( silu(g) * u ), g and u the fp32 results of rows 2i and 2i + 1 (the gated
 *            product fused into the epilogue; silu(t) = t / (1 + exp(-t))).  MATQ_OUT_F32_ACCUM adds the
 *            product to the fp32 values already in y.
 *   workspace device scratch of >= matq_linear_workspace(M, K, N, group) bytes, owned by
 *            the caller, header zero-filled once (see matq_workspace_init).
 * Kernel choice is internal: M <= 16 takes the decode path (persistent TMA-fed streaming
 * kernel, weights unpacked in registers into exact fp16 MMA operands, fp32 accumulation;
 * N <= 2^21); larger M the prefill path (TMA-staged planes dequantised to fp16 tiles in
 * shared memory, tcgen05 MMA with TMEM accumulators).  Input range: the decode path converts
 * x to fp16 operands, exact for |x| in [2^-14, 65504] (smaller values round to fp16's
 * subnormal grid, 2^-24); an activation with |x| >= 65536 sets MATQ_STATUS_XRANGE in the
 * workspace status and leaves that call's y undefined.  The prefill path divides each token's
 * activations by the power of two that keeps its largest value finite in fp16 (exact) and
 * multiplies the token's fp32 results back, so it serves any finite bf16 x; its fp16 weight
 * tiles need |W_hat| below 65504.  Kernels are launched with programmatic
 * dependent launch, so a call may start streaming weights while the previous kernel in the
 * stream finishes; it reads x and writes y only after that kernel completes. */
int matq_linear(const void* x, int M, int K,
                const void* planes, int r_keep,
                const uint16_t* scales, const uint8_t* zeros, int N,
                int r, int group,
                void* y, int y_mode,
                void* workspace, size_t ws_bytes, void* stream);

/* ---- rounded slicing: strict MatQuant and Extra-Precision MatQuant ----------------------- */

/* "Matryoshka Quantization | Summary" §3.2 slices a parent code by rounding instead of
 * truncating:
 *     L = floor(q / 2^(8-r) + 1/2)            (0 <= L <= 2^r; ties round up)
 *     strict MatQuant:          L_c = min(L, 2^r - 1),  W_hat = s * (L_c * 2^(8-r) - z)
 *     Extra-Precision MatQuant: (same page, §7 Errata) no clamp, W_hat = s * (L * 2^(8-r) - z),
 *                               2^r + 1 levels; the top one needs an extra bit for the few
 *                               weights whose codes round up past the last r-bit level.
 * Rounding needs code bit 7 - r besides the r-bit prefix, so libmatq extracts such a slice
 * once from a parent pack into
 *   - a width-r "level pack": MATQ-PL1 planes of width r holding L_c where a code's prefix sits
 *     (r bits per weight), served by matq_linear_rounded with no centring offset;
 *   - the overflow list: for each row n, the inputs k (ascending) whose L = 2^r, in CSR form
 *     (row_ptr [N + 1] int32, cols uint16).  Extra-Precision adds s * 2^(8-r) * x[m, k] to
 *     y[m, n] for each listed weight (on the prefill path the listed weights' tile values
 *     become s * (256 - z) instead).
 * r = 8 rounds nothing: its level pack equals the parent's width-8 planes, its list is empty. */

/* Scratch bytes matq_round_extract needs (4 bytes per (row, 256-input chunk)); 0 if invalid. */
size_t matq_round_scratch_bytes(int N, int K);

/* Extract the width-r rounded slice of a pack (asynchronous on `stream`).
 *   planes   parent pack (matq_pack) with r_keep >= the width whose planes hold code bit 7 - r:
 *            3 for r = 2, 4 for r = 3, 6 for r = 4, 8 for r = 6 and 8 (MATQ_ETRUNC otherwise).
 *   levels   device buffer of >= matq_packed_bytes(N, K, r) bytes (levels_bytes); written with
 *            the clamped levels L_c as a width-r pack.
 *   row_ptr  device [N + 1] int32; written: row n's listed weights are
 *            cols[row_ptr[n] .. row_ptr[n + 1]); row_ptr[N] is the list's length.
 *   cols     device uint16 [cols_cap], or NULL.  NULL: only levels and row_ptr are written;
 *            read row_ptr[N], allocate cols and call again.  Entries at positions >= cols_cap
 *            are not written.  The kernels that read the list load it in aligned 8-entry
 *            blocks, so cols must have room for row_ptr[N] rounded up to a multiple of 8.
 *   scratch  device buffer of >= matq_round_scratch_bytes(N, K) bytes (scratch_bytes).
 * Shapes: K <= 65536 (uint16 inputs) and N * K < 2^31.  Errors: MATQ_EINVAL_R, MATQ_ETRUNC,
 * MATQ_EINVAL_SHAPE, MATQ_ENULL, MATQ_EALIGN, MATQ_ESIZE, MATQ_EDEVICE, MATQ_ECUDA. */
int matq_round_extract(const void* planes, int N, int K, int r_keep, int r,
                       void* levels, size_t levels_bytes,
                       int32_t* row_ptr, uint16_t* cols, size_t cols_cap,
                       void* scratch, size_t scratch_bytes, void* stream);

/* Workspace bytes matq_linear_rounded needs: matq_linear_workspace, plus (M <= 16) room for
 * an fp32 copy of the dense result [M, N] that the list correction starts from. */
size_t matq_linear_rounded_workspace(int M, int K, int N, int group);

/* y = x . W_hat^T for a rounded slice (arguments, output modes, workspace rules and input
 * range as matq_linear, with the level pack in place of the planes and r_keep = r).
 *   row_ptr, cols  the overflow list from matq_round_extract: Extra-Precision MatQuant.
 *                  Both NULL: strict MatQuant (the clamped levels alone).  One NULL: MATQ_ENULL.
 * M <= 16: the decode kernel on the level pack (fp32 result in y, or in the workspace for
 * bf16 and gated outputs), then one correction kernel that adds the listed weights' terms and
 * writes y.  M > 16: the prefill kernel, whose dequantising warps overwrite the listed weights'
 * fp16 tile values; one launch (plus the activation conversion).
 * Bytes read per call: r * N * K / 8 of levels, the scales and zeros, and 2 bytes per listed
 * weight (plus row_ptr). */
int matq_linear_rounded(const void* x, int M, int K,
                        const void* levels, int r,
                        const uint16_t* scales, const uint8_t* zeros, int N, int group,
                        const int32_t* row_ptr, const uint16_t* cols,
                        void* y, int y_mode,
                        void* workspace, size_t ws_bytes, void* stream);

/* ---- the sliced linear layer without a caller workspace -------------------------------- */

/* Capacity, in bytes, of the scratch array that libmatq itself holds for matq_linear_noalloc
 * (one array per device, in static device memory). */
#define MATQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/* matq_linear with the scratch held by libmatq instead of a caller workspace.  This entry
 * point is a library convenience; the sliced-quantisation papers have no counterpart of it.
 *
 * Who needs it: callers that must not allocate device memory at call time and have none to
 * spare for a workspace: a host runtime or plugin that owns every allocation itself and
 * hands the library only its tensors; serving loops where cudaMalloc/cudaFree (which may
 * synchronise the device, and may fail once memory is fragmented) are banned on the hot
 * path; C callers without a memory allocator of their own.  The call allocates nothing on
 * the device or the host, through CUDA or any other library; its scratch is a fixed
 * MATQ_NOALLOC_SCRATCH_BYTES array in libmatq's static device memory.
 *
 * Arguments, output and kernels are those of matq_linear (same results), except:
 *   status_out  optional (NULL: not reported) device pointer to one int, 4-byte aligned.
 *               After the call completes on the device it holds 0, or the device-side
 *               wait-timeout code of this call (then y is undefined).
 *   no workspace arguments.
 * Limits: the sizes must fit the fixed scratch: the smallest workspace matq_linear accepts for
 * them (below) must be <= MATQ_NOALLOC_SCRATCH_BYTES; larger calls return MATQ_ESCRATCH and
 * launch nothing.
 * Every M <= 16 (decode path) fits; M > 16 (prefill path) fits while 262,400 + M*K*2 + M*4
 * bytes (the last two each rounded up to 256) do, e.g. M <= 991 at K = 4096; such a call runs
 * without K splits.  Use matq_linear with a caller workspace beyond that.
 * Set-up: the first call on each device, made with that device current, looks up the device
 * address of the array (cudaGetSymbolAddress; this can load libmatq's device code onto the
 * device) and caches it; a failure returns MATQ_ECUDA.  Make that first call before any
 * stream capture is started on the device.
 * State: unlike the other entry points, this one keeps state between calls: the array and
 * its cached address.
 * Sharing: every call on a device uses the same array, which keeps its last contents; each
 * call first clears the part that must start at zero (an asynchronous memset of the header
 * on `stream`), then launches the kernel, then copies the status word (if status_out).
 * Calls whose executions overlap on the device (different streams, not ordered with one
 * another, or different host threads with such streams) race on the array and give wrong
 * results: order them (one stream, or events).  A cudaDeviceReset invalidates the cached
 * address; do not call this entry point on that device afterwards in the same process. */
int matq_linear_noalloc(const void* x, int M, int K,
                        const void* planes, int r_keep,
                        const uint16_t* scales, const uint8_t* zeros, int N,
                        int r, int group,
                        void* y, int y_mode,
                        int* status_out, void* stream);

/* ---- parent-code choice for several widths -------------------------------------------- */

/* Reconstruction rules a code choice can score with ("MatGPTQ" App. A.1). */
#define MATQ_SLICE_TRUE_PREFIX 0   /* q_hat = p * 2^(8-r) + (2^(8-r) - 1) / 2 (centred)     */
#define MATQ_SLICE_TRUNCATE    1   /* q_hat = p * 2^(8-r) (raw MSB truncation)               */

/* matq_choose_codes -- the parent code of every weight, chosen for several widths at once
 * ("MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models", §3.2 item 2 and
 * App. A.2, Algorithm 2: the quant_MatGPTQ step).  Each weight w[n][k] gets the code q in
 * [0, 255] that minimises
 *     total(q) = sum_i lambdas[i] * (w - s * (q_hat_{widths[i]}(q) - z))^2
 * with s, z the weight's group scale and zero point and q_hat the rule of slice_mode.  The
 * arithmetic is fp32 with every operation rounded on its own (s * (q_hat - z) is exact; then
 * e = w - that, e * e, lambda * (e * e), and the running sum, terms added in the order of
 * `widths`), the precision the page gives for its candidate errors; on a tie the smallest
 * code wins (the first minimum of an argmin over q = 0..255).  Non-finite inputs or s <= 0
 * follow the same definition (an argmin meeting NaN totals takes the first NaN).
 * The page runs this per column inside GPTQ, on weights that error feedback has updated;
 * this call applies it to a whole matrix as given (the Hessian pass that produces those
 * weights needs calibration data and is not part of libmatq).  With MATQ_SLICE_TRUE_PREFIX
 * and a positive weight on width 8 the result is round-to-nearest (cell boundaries of every
 * width fall half way between two codes); raw truncation makes the widths trade off.
 *   w        fp32 [N, K] row-major (device).
 *   scales   fp16 [N, K/group], zeros uint8 [N, K/group] (device), as matq_linear takes them.
 *   group    64 or 128; K a positive multiple of group (K need not be a multiple of 256).
 *   n_widths 1..5; widths: HOST array, strictly ascending, each in {2, 3, 4, 6, 8}.
 *   lambdas  HOST array of n_widths finite, non-negative weights (the pages do not print the
 *            values they used; equal weights summing to one are a neutral choice).
 *   codes    uint8 [N, K] (device): the chosen parent codes, ready for matq_pack.
 * Errors: MATQ_EINVAL_GROUP, MATQ_EINVAL_SHAPE, MATQ_ENULL, MATQ_EINVAL_R (widths),
 * MATQ_EINVAL_ARG (lambdas, slice_mode), MATQ_EALIGN, MATQ_EDEVICE, MATQ_ECUDA. */
int matq_choose_codes(const float* w, int N, int K,
                      const uint16_t* scales, const uint8_t* zeros, int group,
                      int n_widths, const int* widths, const float* lambdas, int slice_mode,
                      uint8_t* codes, void* stream);

/* ---- glue of the Mix'n'Match FFN stack ------------------------------------------------- */

/* n = bf16( h / sqrt(mean(h^2) + eps) ) row by row (unit-gain RMSNorm).
 *   h [M, D] fp32, n_out [M, D] bf16. */
int matq_rmsnorm(const float* h, int M, int D, float eps, void* n_out, void* stream);

/* a = bf16( silu(gate) * up ), silu(t) = t / (1 + exp(-t)), computed in fp32.
 *   gate, up, a_out [M, F] bf16. */
int matq_silu_mul(const void* gate, const void* up, int M, int F, void* a_out, void* stream);

/* The same product for the output of ONE fused gate+up projection (gate and up read the same
 * x, so their weights can be packed as one [2F, D] matrix and served by one matq_linear call;
 * "MatGPTQ" §4 applies the sliced kernel per linear layer, this fusion is this library's).
 *   gu    [M, 2F] bf16: row m holds gate in columns 0..F-1 and up in columns F..2F-1.
 *   a_out [M, F] bf16: a = bf16( silu(gate) * up ).  F % 8 == 0 takes the vector path. */
int matq_silu_mul_gu(const void* gu, int M, int F, void* a_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MATQ_H */
