/*
 * twell.h -- C ABI of libtwell.so: the activation-sparse gated FFN of a
 * ReLU-gated transformer layer on one NVIDIA B200 (sm_100a), with the
 * activations carried in the Tile-wise ELLPACK ("TwELL") format.
 *
 * Method: technical summary page of "Sparser, Faster, Lighter Transformer
 * Language Models" (arXiv 2603.23198):
 *   section 2.1  TwELL format, built in the gate matmul's epilogue in shared
 *                memory, g = ReLU(x Wg);
 *   section 2.2  fused up + down projection over the non-zero activations;
 *   section 2.3  hybrid format for training (compact ELL + dense backup rows);
 *   section 2.4  hybrid-to-dense / dense-to-hybrid training kernels with an
 *                L1 term on the gate activations.
 *
 * Conventions for every entry point
 * ---------------------------------
 * Ownership   The caller owns every buffer.  The library never allocates or
 *             frees device memory and never keeps a pointer after the call.
 * Pointers    All tensor pointers are DEVICE pointers, 16-byte aligned.
 * Layouts     Row-major.  x, y, dy, dx: [T][d].  Weights: [F][d] with row j =
 *             unit j's d-vector: Wg_t = gate_proj.weight, Wu_t = up_proj.weight,
 *             Wd = down_proj.weight transposed ([F][d]).  The dense comparator
 *             alone takes the down weight as down_proj.weight ([d][F]).
 * dtypes      TW_BF16 tensors are raw bf16; TW_F32 tensors are IEEE fp32.
 *             Arithmetic accumulates in fp32.
 * Asynchrony  Work is enqueued on `stream` and the call returns without
 *             synchronising.  Pass 0 for the legacy default stream.
 * Errors      The return value reports host-side validation (checked before
 *             any launch) and launch errors.  Conditions found on the device
 *             (capacity exceeded, a pipeline wait that timed out) are OR-ed
 *             into the caller's `dev_status` word as bit (1 << tw_status);
 *             dev_status may be NULL.  The caller zeroes it and reads it after
 *             synchronising; tw_status_string names each code.
 * Limits      W in {64, 128, 256}; 0 <= C <= W; F % W == 0; d % 8 == 0; 8 <= d <= 2048
 *             (bf16 rows) or d <= 1024 (fp32 rows) for the fused and hybrid
 *             kernels; T >= 0.  With T == 0 the arrays sized by T (x, y, dy,
 *             dx, the TwELL and hybrid per-token arrays, the workspaces) may
 *             be NULL: the calls only reset spill_n / n_backup and write zero
 *             weight gradients.  F <= 65536 (hybrid
 *             indices are uint16); for hybrid arguments F % 8 == 0 and
 *             F <= 51200.
 */
#ifndef TWELL_H
#define TWELL_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define TW_API __attribute__((visibility("default")))
#else
#define TW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TW_OK = 0,
  TW_ERR_INVALID_ARG = 1,      /* null pointer, bad size, mismatched shapes   */
  TW_ERR_UNSUPPORTED = 2,      /* valid but outside the limits above          */
  TW_ERR_ALIGNMENT = 3,        /* a pointer is not 16-byte aligned            */
  TW_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed        */
  TW_ERR_SPILL_CAPACITY = 5,   /* device: more TwELL spill entries than cap   */
  TW_ERR_BACKUP_CAPACITY = 6,  /* device: more hybrid backup rows than cap    */
  TW_ERR_TIMEOUT = 7,          /* device: a bounded pipeline wait ran out     */
  TW_ERR_WORKSPACE = 8         /* workspace smaller than the size query says  */
} tw_status;

typedef enum { TW_F32 = 0, TW_BF16 = 1 } tw_dtype;

/*
 * TwELL tensor for the gate activations g [T][F] (section 2.1): the F columns
 * are cut into K = F / W tiles of width W.  For every (tile k, token t):
 *   cnt[k][t]        number of non-zero g in columns [k*W, (k+1)*W) -- the
 *                    true count, which may exceed C;
 *   val[k][t][s], idx[k][t][s], s < min(cnt, C)
 *                    the first non-zeros in ascending column order and their
 *                    tile-local column (0..W-1); slots s >= cnt hold (+0, 0);
 *   if cnt > C       the whole W-wide segment is copied to spill entry
 *                    r = spill_ref[k][t]: spill_val[r][0..W-1], and
 *                    spill_tk[r] = {t, k}.  Entries are numbered in arrival
 *                    order (not deterministic); *spill_n receives the number
 *                    of entries needed, which may exceed spill_cap (entries
 *                    past the cap are dropped and TW_ERR_SPILL_CAPACITY is
 *                    flagged).  spill_ref is written only where cnt > C.
 * Array shapes: val [K][T][C] (dtype), idx [K][T][C] uint8, cnt [K][T] uint8,
 * spill_ref [K][T] int32, spill_tk [spill_cap][2] int32, spill_val
 * [spill_cap][W] (dtype), spill_n one int32.  With C == 0 val/idx may be NULL.
 * A uint8 count holds 0..255: a 256-wide tile whose 256 units are all active
 * is stored with cnt = 255 and flags TW_ERR_UNSUPPORTED in dev_status (its
 * spilled segment, when C < 256, still holds every value).
 */
typedef struct {
  int32_t T, F, W, C;
  tw_dtype dtype;
  void* val;
  uint8_t* idx;
  uint8_t* cnt;
  int32_t* spill_ref;
  int32_t spill_cap;
  int32_t* spill_tk;
  void* spill_val;
  int32_t* spill_n;
} tw_twell;

/*
 * Hybrid tensor (section 2.3): every token row is either an ELL row or a
 * dense backup row, decided by its non-zero count nnz = row_nnz[t]:
 *   nnz <= C_h   ELL row: row_slot[t] = -1; ell_g[t][0..nnz) are its
 *                non-zeros in ascending unit order, ell_idx the global unit
 *                indices; slots past nnz hold (+0, 0);
 *   nnz >  C_h   backup row: row_slot[t] = b, its slot; backup_rows[b] = t;
 *                backup_g[b][0..F) is the dense g row.  Slots are numbered in
 *                ascending token order.  *n_backup receives the number of
 *                backup rows needed (rows past backup_cap are dropped and
 *                TW_ERR_BACKUP_CAPACITY is flagged).
 * ell_u / backup_u hold the up activation u = x Wu on the same pattern (+0
 * elsewhere in ell_u and in the stored backup rows, the first
 * min(*n_backup, backup_cap); rows past those are not written);
 * hybrid_ffn_forward fills them and the backward reads them.
 * Shapes: ell_g, ell_u [T][C_h] (dtype); ell_idx [T][C_h] uint16; row_nnz,
 * row_slot [T] int32; backup_rows [backup_cap] int32; backup_g, backup_u
 * [backup_cap][F] (dtype); n_backup one int32.
 */
typedef struct {
  int32_t T, F, C_h;
  tw_dtype dtype;
  void* ell_g;
  void* ell_u;
  uint16_t* ell_idx;
  int32_t* row_nnz;
  int32_t* row_slot;
  int32_t backup_cap;
  int32_t* backup_rows;
  void* backup_g;
  void* backup_u;
  int32_t* n_backup;
} tw_hybrid;

/*
 * Gate projection with TwELL output (section 2.1): g = ReLU(x Wg), with
 * z = x Wg accumulated in fp32 and g rounded to out->dtype, packed straight
 * into *out by the matmul's epilogue.  x [T][d] and Wg_t [F][d] have `dtype`,
 * which must equal out->dtype.  bf16 runs on the tcgen05 tensor cores fed by
 * TMA (for T <= 64 with the d reduction split over a thread-block cluster,
 * summed in a fixed order); fp32 runs at full fp32 precision on the CUDA
 * cores.  out->T, out->F
 * must equal T, F.  g_dense_dump, if not NULL, receives the dense rounded g
 * [T][F] (dtype) -- a test aid; pass NULL for speed.
 */
TW_API tw_status twell_gate_gemm(const void* x, const void* Wg_t, int32_t T, int32_t d, int32_t F,
                          tw_dtype dtype, const tw_twell* out, void* g_dense_dump,
                          int32_t* dev_status, cudaStream_t stream);

/* Bytes of workspace twell_fused_updown needs for T tokens of width d. */
TW_API size_t twell_fused_updown_workspace_size(int32_t T, int32_t d);

/*
 * Fused up + down projection over TwELL (section 2.2): for every token t and
 * every active unit j of g (slots and spilled segments),
 *   u = x_t . Wu_t[j]  (fp32),  h = g_tj * u,  y_t += h * Wd[j]  (fp32),
 * and y_t is stored in y_dtype.  No dense intermediate reaches memory.
 * x, Wu_t and Wd have g->dtype.  y [T][d].
 * ws: device workspace of at least twell_fused_updown_workspace_size(T, d)
 * bytes (a work plan, and fp32 partial rows for tokens whose active units are
 * split over several warps).  Its counters are cleared on `stream` by the
 * call's own kernels; calls that share one workspace must not overlap on the
 * device (calls queued one after another on one stream do not).  y is
 * deterministic: partial rows are summed in a fixed order.
 */
TW_API tw_status twell_fused_updown(const void* x, const tw_twell* g, const void* Wu_t,
                             const void* Wd, int32_t d, void* y, tw_dtype y_dtype, void* ws,
                             size_t ws_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * twell_fused_updown without a workspace argument.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- for example a plugin whose host framework forbids device
 * allocation in its call path, or a serving process that handed all device
 * memory to its own pool at start-up.  It computes the same y (same
 * kernels) with its work plan in a 16 MiB array inside the library's device
 * image, held on every GPU that loads the library until the process exits.
 *   - No cudaMalloc or cudaFree is called; the caller passes inputs and
 *     outputs exactly as for twell_fused_updown.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it for the life of the process; make
 *     that first call before any stream capture, and do not use the entry
 *     point across cudaDeviceReset (the cached address would be stale).
 *   - The plan of T tokens must fit 16 MiB, about 24 bytes per token: T up to
 *     696,848 fits for every supported d; a T whose plan does not fit returns
 *     TW_ERR_UNSUPPORTED before any device work.  The rest of the array holds
 *     partial rows of split tokens; when fewer heavy tokens can be split than
 *     the workspace version would split, the rest run unsplit: y is the same
 *     up to fp32 summation order.
 *   - Arguments are checked as for twell_fused_updown; with T == 0 the
 *     token-sized buffers (x, y and the TwELL per-token arrays) may be NULL
 *     and the call returns TW_OK without device work.
 *   - Every call shares the one array, and the call clears the part that must
 *     start at zero.  Calls whose work overlaps on the GPU (different streams
 *     or host threads without ordering) race on it and give wrong results.
 */
TW_API tw_status twell_fused_updown_noalloc(const void* x, const tw_twell* g, const void* Wu_t,
                                            const void* Wd, int32_t d, void* y, tw_dtype y_dtype,
                                            int32_t* dev_status, cudaStream_t stream);

/*
 * The whole FFN of a small batch -- decoding, 1 <= T <= 64 tokens -- in ONE
 * launch (sections 2.1 and 2.2): g = ReLU(x Wg) packed into *g as
 * twell_gate_gemm packs it, then y = sum over the active units of
 * g (x . Wu_t[j]) Wd[j], as twell_fused_updown computes it (fp32 accumulation,
 * deterministic).  bf16 only, g->W == 128, 64 <= d <= 2048, d % 8 == 0.
 * A small batch is bound by streaming Wg from HBM; separate gate and fused
 * launches spend more on launches and set-up than on that stream, so this
 * call runs one persistent cooperative grid (one CTA per SM) whose phases
 * are separated by grid-wide barriers.  g_dense_dump as in twell_gate_gemm.
 * ws: at least twell_ffn_small_batch_workspace_size(T, d, F) bytes.  Its
 * first 256 bytes are barrier counters that must be zero when a call starts:
 * allocate the workspace zero-filled once; every call leaves them at zero
 * (after a call that flagged TW_ERR_TIMEOUT, zero them again).  Calls that
 * share one workspace must not overlap on the device.  The launch fails with
 * TW_ERR_CUDA if the device cannot hold one CTA per SM for a cooperative
 * launch.
 */
TW_API size_t twell_ffn_small_batch_workspace_size(int32_t T, int32_t d, int32_t F);
TW_API tw_status twell_ffn_small_batch(const void* x, const void* Wg_t, const void* Wu_t,
                                       const void* Wd, int32_t T, int32_t d, int32_t F,
                                       const tw_twell* g, void* g_dense_dump, void* y,
                                       tw_dtype y_dtype, void* ws, size_t ws_bytes,
                                       int32_t* dev_status, cudaStream_t stream);

/*
 * TwELL -> hybrid conversion (section 2.3).  out->T, out->F equal g->T,
 * g->F and out->dtype equals g->dtype.  Fills ell_g, ell_idx, row_nnz,
 * row_slot, backup_rows, backup_g, n_backup.
 */
TW_API tw_status twell_to_hybrid(const tw_twell* g, const tw_hybrid* out, int32_t* dev_status,
                          cudaStream_t stream);

/* Bytes of workspace hybrid_ffn_forward needs for T tokens of width d. */
TW_API size_t hybrid_ffn_forward_workspace_size(int32_t T, int32_t d);

/*
 * Training forward on the hybrid pattern (sections 2.3-2.4): u = x Wu sampled
 * at the active positions -> gu->ell_u / gu->backup_u (rounded to gu->dtype,
 * +0 off the pattern), then y = (g * u) Wd with fp32 accumulation and the
 * unrounded u.  x, Wu_t, Wd have gu->dtype.  y [T][d] in y_dtype.
 * ws: device workspace of at least hybrid_ffn_forward_workspace_size bytes
 * (the same work plan as twell_fused_updown; calls sharing one workspace must
 * not overlap on the device).
 */
TW_API tw_status hybrid_ffn_forward(const void* x, const tw_hybrid* gu, const void* Wu_t,
                             const void* Wd, int32_t d, void* y, tw_dtype y_dtype, void* ws,
                             size_t ws_bytes, int32_t* dev_status, cudaStream_t stream);

/* Bytes of workspace hybrid_ffn_backward needs for these sizes. */
TW_API size_t hybrid_ffn_backward_workspace_size(int32_t T, int32_t d, int32_t F, int32_t C_h,
                                          int32_t backup_cap);

/*
 * Training backward on the hybrid pattern (section 2.4), for the loss
 * L = sum(y * dy) + l1_lambda * sum(g), from the saved g and u of gu:
 * for every active (t, j):  dh = dy_t . Wd[j];  du = dh * g;
 * dz = dh * u + l1_lambda;  dx_t += du Wu_t[j] + dz Wg_t[j];
 * dWd[j] += (g u) dy_t;  dWu_t[j] += du x_t;  dWg_t[j] += dz x_t.
 * Inactive positions contribute nothing (ReLU'(0) = 0, sign(0) = 0).
 * dx [T][d] in dx_dtype; dWg_t, dWu_t, dWd [F][d] fp32, fully overwritten.
 * Weight gradients are summed in ascending token order (deterministic).
 * ws: device workspace of at least hybrid_ffn_backward_workspace_size bytes.
 */
TW_API tw_status hybrid_ffn_backward(const void* x, const void* dy, const tw_hybrid* gu,
                              const void* Wg_t, const void* Wu_t, const void* Wd, int32_t d,
                              float l1_lambda, void* dx, tw_dtype dx_dtype, float* dWg_t,
                              float* dWu_t, float* dWd, void* ws, size_t ws_bytes,
                              int32_t* dev_status, cudaStream_t stream);

/*
 * Dense comparator (the non-sparse baseline of section 4), bf16 only, on the
 * same tcgen05 pipeline: h = ReLU(x Wg) * (x Wu) in one GEMM over the
 * interleaved gate/up weights, written to h_ws [T][F] bf16, then y = h Wd
 * with Wd_dense = down_proj.weight [d][F].  y [T][d] bf16.
 */
TW_API tw_status dense_ffn_forward(const void* x, const void* Wg_t, const void* Wu_t,
                            const void* Wd_dense, int32_t T, int32_t d, int32_t F, void* h_ws,
                            void* y, int32_t* dev_status, cudaStream_t stream);

/*
 * Dense training comparator (the non-sparse baseline of the training results
 * of section 4), bf16 only, on the same tcgen05 pipeline and with the same
 * weight layouts as the sparse path (Wg_t, Wu_t, Wd all [F][d]).  One training
 * step of the gated FFN for the loss L = sum(y * dy) + l1_lambda * sum(g):
 *   forward   z = x Wg, u = x Wu, g = ReLU(z), h = g u, y = h Wd (y fp32);
 *   backward  dh = dy Wd^T, du = dh g, dz = (dh u + l1_lambda) where g > 0,
 *             dx = du Wu^T + dz Wg^T (fp32), and the fp32 weight gradients
 *             dWd = h^T dy, dWu_t = du^T x, dWg_t = dz^T x ([F][d]).
 * g, u, h are stored bf16 (g rounded first, as the sparse path stores it);
 * du and dz are rounded to bf16 as the operands of the dx and weight-gradient
 * matmuls.  d % 32 == 0, d >= 64, F % 128 == 0, any T >= 0.
 * ws: at least dense_ffn_train_workspace_size(T, F) bytes: g, u, h [T][F]
 * bf16 (the activations the forward saves for the backward,
 * dense_ffn_train_saved_bytes(T, F) bytes) followed by du, dz [T][F] bf16
 * (backward scratch).  The backward reads what the forward saved in the same
 * workspace; calls sharing it must not overlap on the device.
 */
TW_API size_t dense_ffn_train_workspace_size(int32_t T, int32_t F);
TW_API size_t dense_ffn_train_saved_bytes(int32_t T, int32_t F);
TW_API tw_status dense_ffn_train_forward(const void* x, const void* Wg_t, const void* Wu_t,
                                         const void* Wd, int32_t T, int32_t d, int32_t F,
                                         void* ws, size_t ws_bytes, float* y,
                                         int32_t* dev_status, cudaStream_t stream);
TW_API tw_status dense_ffn_train_backward(const void* x, const void* dy, const void* Wg_t,
                                          const void* Wu_t, const void* Wd, int32_t T, int32_t d,
                                          int32_t F, float l1_lambda, void* ws, size_t ws_bytes,
                                          float* dx, float* dWg_t, float* dWu_t, float* dWd,
                                          int32_t* dev_status, cudaStream_t stream);

/*
 * Test aid for the bounded pipeline waits; not needed in normal use.  The
 * next twell_gate_gemm call that runs the tile GEMM (T > 64, or any T when
 * W != 128) withholds its TMA loads and bounds its waits by wait_limit_ns:
 * the MMA issuer's first wait can then never complete, so every CTA must give
 * up after about wait_limit_ns, flag TW_ERR_TIMEOUT in dev_status, stop its
 * roles, free its tensor memory and return (nothing is in flight, since
 * nothing was issued).  The TwELL output of that call is not written.  The
 * setting is consumed by that one call; later calls run normally.
 */
TW_API void tw_test_withhold_next_gate_loads(uint64_t wait_limit_ns);

/* Human-readable name of a status code. */
/* Measurement aid, not part of the FFN: the gathered-row rate of the fused
 * up + down projection's roofline.  n_gathers rows of the bf16 matrix
 * mat [rows][d] are read in full with 16-byte loads, gather i taking row
 * splitmix64((seed << 32) ^ i) mod rows (splitmix64 as published by Steele,
 * Lea and Flood, 2014), by the warps of a persistent grid (one CTA of 16
 * warps per SM, two rows in flight per warp).
 * checksum: device word, zeroed by the caller, receives the XOR of every
 *           32-bit word read (so the loads happen and the result can be
 *           checked on the host, whatever the order).
 * Limits: rows >= 1, 8 <= d <= 2048, d % 8 == 0, n_gathers >= 0; mat
 * 16-byte aligned.  n_gathers == 0 launches nothing. */
TW_API tw_status tw_measure_row_gather(const void* mat, int32_t rows, int32_t d,
                                       int64_t n_gathers, uint32_t seed, uint32_t* checksum,
                                       cudaStream_t stream);

/* Measurement aid, not part of the FFN: the floor of a launch that streams a
 * small-batch step's bytes.  The device buffer buf is read once, front to
 * back, with 16-byte loads (two CTAs of 512 threads per SM, eight loads in
 * flight per thread) by one launch.  Timed with a cold L2 on the gate's
 * weight bytes, it is what that launch costs with nothing else to do.
 * checksum: device word, zeroed by the caller, receives the XOR of every
 *           32-bit word read.
 * Limits: bytes >= 0 and a multiple of 16; buf 16-byte aligned.  bytes == 0
 * launches nothing. */
TW_API tw_status tw_measure_stream_read(const void* buf, int64_t bytes, uint32_t* checksum,
                                        cudaStream_t stream);

TW_API const char* tw_status_string(tw_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
TW_API int32_t twell_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TWELL_H */
