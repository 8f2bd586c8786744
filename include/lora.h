/*
 * lora.h - C ABI of the B200 (sm_100a) fused LoRA linear layer library.
 *
 * The layer (fastaf 0.1.0, "Minimal LoRA fine-tuning with hand-written
 * Triton kernels", section "FWD kernel speedup"):
 *
 *     Y = X W^T + s (X A^T) B^T,        s = alpha / r
 *
 * its backward for a frozen W (same page, section "BWD kernel speedup",
 * which names the dA, dB and dX kernels; the formulas follow from the
 * forward by the chain rule), with T = X A^T recomputed (or kept from the
 * forward through lora_fwd_save and LORA_BWD_T_SAVED):
 *
 *     dT = s dY B,   dB = s dY^T T,   dA = dT^T X,   dX = dY W + dT A
 *
 * and the adapter merge of the unsloth fork commit log
 * (scripts/benchmarks/qwen3_flex_inference.py, the commit replacing
 * copy + merge_adapter by one addmm(pristine, B, A, alpha=scaling)):
 *
 *     W_dst = W_src + s B A      (fp32 accumulate, one rounding to bf16)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are bf16 (passed as raw bit buffers), row-major, contiguous:
 *   X[M, d_in], W[d_out, d_in], A[r, d_in], B[d_out, r], Y[M, d_out],
 *   dY[M, d_out], dX[M, d_in], dA[r, d_in], dB[d_out, r].
 * - All tensor pointers are DEVICE pointers on the current CUDA device,
 *   16-byte aligned.  Pointers to tensors with a zero-sized M dimension
 *   (X, Y, dY, dX, and the workspace) may be NULL when M == 0.  The caller
 *   allocates and owns every buffer and the stream; the library never calls
 *   cudaMalloc.  Its GPU module holds a fixed amount of static device memory
 *   on every device that loads it: a status word, the forward's exchange
 *   slots (8 x about 4 MiB, see lora_fwd) and the scratch of
 *   lora_bwd_noalloc (32 MiB).
 * - d_in and d_out are multiples of 8 (16-byte row pitch); r is a multiple
 *   of 8 in [8, 128]; M >= 0 (M = 0 is a no-op).  Row counts need not be
 *   multiples of any tile size.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *   asynchronous with respect to the host and ordered on `stream`.
 * - s = alpha / r is computed in fp32 on the host (the *_scaled forms below
 *   take s itself instead of alpha).
 * - Outputs must not overlap inputs, except W_dst == W_src in lora_merge.
 * - Argument errors are returned before anything is launched and leave no
 *   side effects.  A failed launch returns LORA_ERR_CUDA.  Kernels bound
 *   every wait; a wait that runs out sets a device-side status word that
 *   lora_get_device_status() reports (LORA_ERR_TIMEOUT).
 * - Only sm_100 devices (B200) are supported; others get
 *   LORA_ERR_UNSUPPORTED_DEVICE.
 * - Calls on different streams may run concurrently.  Besides the
 *   per-device status word, the library's only state shared between calls
 *   is the forward's exchange slots, each bound to one stream (see
 *   lora_fwd).
 * - Kernels are launched with programmatic dependent launch: a kernel's
 *   set-up may overlap the end of the previous kernel on the stream, but it
 *   touches no global memory before that kernel has completed, so stream
 *   order is kept (LORA_B200_PDL=0 in the environment turns this off).
 */
#ifndef LORA_B200_H
#define LORA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LORA_ABI_VERSION 4

typedef enum {
  LORA_OK = 0,
  LORA_ERR_NULL = 1,               /* a required pointer is NULL */
  LORA_ERR_SHAPE = 2,              /* negative size, or d_in/d_out not a multiple of 8 */
  LORA_ERR_ALIGN = 3,              /* a pointer is not 16-byte aligned */
  LORA_ERR_RANK = 4,               /* r not a multiple of 8 in [8, 128] */
  LORA_ERR_WORKSPACE = 5,          /* workspace NULL or smaller than required */
  LORA_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed */
  LORA_ERR_TIMEOUT = 7,            /* a kernel gave up on a bounded wait */
  LORA_ERR_UNSUPPORTED_DEVICE = 8, /* current device is not sm_100 */
  LORA_ERR_ALIAS = 9,              /* an output overlaps an input */
  LORA_ERR_FLAGS = 10              /* a flags argument has an unknown bit set */
} lora_status_t;

/* ABI version of the loaded library (LORA_ABI_VERSION it was built with). */
int lora_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* lora_status_string(lora_status_t status);

/*
 * Forward: Y = X W^T + s (X A^T) B^T, rounded once to bf16.
 *   X[M, d_in], W[d_out, d_in], A[r, d_in], B[d_out, r] in; Y[M, d_out] out.
 * The [M, r] down-projection T = X A^T stays on chip: it is accumulated in
 * tensor memory beside the base product, scaled by s and rounded to bf16
 * (as an unfused bf16 X @ A.T would be), and fed to the up-projection,
 * which accumulates onto the base product before the single store of Y.
 * When the output has few 128 x 128 tiles (small M or a small weight), the
 * contraction is split over the CTAs of a thread-block cluster and the
 * partial sums of T and of the base product are added in a fixed order
 * through distributed shared memory (still on chip, no atomics).
 * Otherwise the tiles are dealt to CTA pairs that walk the output; when
 * several pairs work on rows of the same M block, the first to compute its
 * T publishes s T (bf16, the exact operand of the up-projection) in an
 * exchange slot of library-owned device memory and the others copy it, so
 * that every pair can be kept busy while T is computed about once per M
 * block.  A slot is bound to the stream of the first forward that needs
 * one and serves every later forward on that stream (they run one after
 * another); up to 8 streams per device get one, and a forward on any other
 * stream, or one being captured into a CUDA graph, runs without it (slower,
 * same results).  Y is the same bit for bit with or without the exchange.
 */
lora_status_t lora_fwd(const void* X, const void* W, const void* A, const void* B, void* Y,
                       int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                       void* stream);

/*
 * Forward that also keeps T for the backward (the pages describe the forward
 * and the backward, not what passes between them; keeping T is a choice of
 * this library): Y exactly as lora_fwd (bit for bit), and T = X A^T (unscaled, an fp32 sum rounded once to bf16; zero
 * columns past r) written into `workspace`, a buffer of at least lora_bwd_workspace_size(M, d_in,
 * d_out, r) bytes, 256-byte aligned, that overlaps none of X, W, A, B, Y.
 * Pass the same workspace to lora_bwd_ex or lora_bwd_grads with
 * LORA_BWD_T_SAVED, which then skip recomputing T.  The T slot's layout is
 * the library's own; only the workspace as a whole is passed along.
 * In the tiled forward the tile of N index 0 of every M block stores its
 * rows of T from the epilogue (no extra pass over X): each value is the very
 * sum that the up-projection scales.  In the split-contraction form for
 * small outputs, T is one more launch that reads X and sums in its own
 * order.
 * With M == 0 nothing happens (the workspace may then be NULL).
 */
lora_status_t lora_fwd_save(const void* X, const void* W, const void* A, const void* B, void* Y,
                            int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of device scratch lora_bwd needs for this shape (0 when M == 0).
 * Holds T and dT as bf16 [M, r_pad] (r_pad = r rounded up to 16), each at a
 * 256-byte aligned offset.
 */
size_t lora_bwd_workspace_size(int64_t M, int64_t d_in, int64_t d_out, int32_t r);

/*
 * Backward for frozen W:
 *   dX[M, d_in]  = dY W + dT A       (bf16)
 *   dA[r, d_in]  = dT^T X            (bf16, reduced over M in fp32)
 *   dB[d_out, r] = s dY^T T          (bf16, reduced over M in fp32)
 * with T = X A^T recomputed and dT = s dY B, both rounded to bf16 and kept
 * in the workspace by a first launch; a second launch reduces dA and dB;
 * dX is then one product over the contraction [d_out | r], dY W + dT A,
 * rounded once.
 * `workspace` is caller-owned device memory of at least
 * lora_bwd_workspace_size(...) bytes, 256-byte aligned; its contents on
 * entry do not matter and are clobbered.  Results are bitwise repeatable:
 * the M reduction of dA and dB adds fixed per-split partial sums in a fixed
 * order inside a thread-block cluster, with no atomics.
 * With M == 0, dA and dB are set to zero and nothing else happens.
 */
lora_status_t lora_bwd(const void* X, const void* W, const void* A, const void* B,
                       const void* dY, void* dX, void* dA, void* dB,
                       int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Flags of lora_bwd_ex and lora_bwd_grads. */
#define LORA_BWD_FP32_GRADS 1u /* dA and dB are fp32 (float) instead of bf16 */
#define LORA_BWD_T_SAVED 2u    /* the workspace already holds T from lora_fwd_save */

/*
 * lora_bwd with flags.  flags == 0 is exactly lora_bwd.  With
 * LORA_BWD_FP32_GRADS, dA[r, d_in] and dB[d_out, r] are fp32 buffers (same
 * shapes and layouts, 4 bytes per element, 16-byte aligned) and receive the
 * fp32 reductions over M before any rounding: each value is the one that
 * lora_bwd rounds to bf16 (RNE), so rounding them gives lora_bwd's results
 * bit for bit.  Meant for fp32 optimizer states and for summing per-rank
 * partial gradients in fp32 before a single rounding (data parallelism).
 * With M == 0 they are set to zero.
 * With LORA_BWD_T_SAVED the workspace must hold what a lora_fwd_save call
 * of the same X, A and shape left there (nothing may have written the
 * workspace since): T is not recomputed and the first launch reads dY alone
 * (for dT), one pass over X less.  dB then uses the forward's T, rounded
 * from the forward's own accumulation order, and dT is reduced with its own
 * split of the contraction, so the results agree with those of flags == 0
 * to within bf16 rounding of T and dT, not bit for bit.
 * Other rules as lora_bwd; an unknown flag bit returns LORA_ERR_FLAGS
 * before anything is launched.
 */
lora_status_t lora_bwd_ex(const void* X, const void* W, const void* A, const void* B,
                          const void* dY, void* dX, void* dA, void* dB,
                          int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                          void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);

/*
 * The backward of lora_bwd_ex in two calls on one workspace, for callers
 * that want dA and dB before dX is computed, e.g. to start summing them
 * across data-parallel ranks while dX runs:
 *   lora_bwd_grads: T (unless LORA_BWD_T_SAVED) and dT into the workspace,
 *                   then dA and dB (flags as in lora_bwd_ex);
 *   lora_bwd_dx:    dX = dY W + dT A from the dT that the preceding
 *                   lora_bwd_grads call of the same shape left in
 *                   `workspace`.
 * Called in that order on one stream (or with the second ordered after the
 * first), with the same M, d_in, d_out, r and workspace, and nothing
 * writing the workspace in between, they give exactly lora_bwd_ex's results,
 * bit for bit.  Argument rules as lora_bwd_ex for the tensors each call
 * takes.
 */
lora_status_t lora_bwd_grads(const void* X, const void* A, const void* B, const void* dY, void* dA, void* dB,
                             int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                             void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);
lora_status_t lora_bwd_dx(const void* W, const void* A, const void* dY, void* dX,
                          int64_t M, int64_t d_in, int64_t d_out, int32_t r,
                          const void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward without a workspace argument (the pages describe no such entry
 * point; it is a service of this library, not part of the method).
 *
 * Same arguments, results and rules as lora_bwd, minus `workspace` and
 * `workspace_bytes`.  It is for callers that cannot call cudaMalloc, such
 * as a plugin whose host program owns all device memory through its own
 * pool, or a service loop that must not allocate after start-up because
 * cudaMalloc can wait for the device to go idle and can fail under memory
 * pressure.  Instead of a caller workspace it uses a fixed 32 MiB scratch
 * array that the library reserves in device global memory on every GPU
 * that loads it, for the life of the process.
 *  - Shapes whose lora_bwd_workspace_size(...) exceeds 32 MiB are refused
 *    with LORA_ERR_WORKSPACE (and a message on stderr) before any launch.
 *  - The first call on each device looks up the array's device address
 *    (with that device current) and keeps it; make that first call before
 *    any stream capture begins.  After a device reset (a new context) the
 *    next call looks it up again, so it too should come before a capture.
 *  - All calls share the one array and it keeps the last call's contents;
 *    nothing in it needs to start at zero.  Calls whose work can overlap on
 *    the GPU (e.g. on two streams) race on it: keep them on one stream.
 *  - Allocates no device memory.
 */
lora_status_t lora_bwd_noalloc(const void* X, const void* W, const void* A, const void* B,
                               const void* dY, void* dX, void* dA, void* dB,
                               int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                               void* stream);

/*
 * Merge: W_dst[d_out, d_in] = bf16_rne(W_src + s * (B A)), the rank-r
 * product accumulated in fp32 and rounded once.  W_src is the pristine base
 * (restore + merge in one pass) or W_dst itself (in place).
 * A[r, d_in], B[d_out, r].
 */
lora_status_t lora_merge(const void* W_src, const void* A, const void* B, void* W_dst,
                         int64_t d_out, int64_t d_in, int32_t r, float alpha, void* stream);

/* One matrix of a batched merge (all pointers device pointers). */
typedef struct {
  const void* W_src;
  const void* A;
  const void* B;
  void* W_dst;
  int64_t d_out;
  int64_t d_in;
} lora_merge_desc_t;

/*
 * Batched merge of n matrices sharing r and alpha (e.g. every LoRA target of
 * a model), one persistent launch.  `descs` is a HOST array of n entries,
 * read during the call.  Each entry follows lora_merge's rules.
 */
lora_status_t lora_merge_batched(const lora_merge_desc_t* descs, int32_t n, int32_t r,
                                 float alpha, void* stream);

/*
 * Grouped forward: n independent forwards sharing r and alpha in one launch,
 * for the launch-bound regime of many small layers (fastaf 0.1.0, "FWD
 * kernel speedup": below the overhead threshold, launch overhead dominates
 * small batches; e.g. the q, k and v projections of one input, or the
 * adapters of several requests).  Each entry is one lora_fwd problem with
 * lora_fwd's rules (entries with M = 0 are skipped).  No entry's Y may
 * overlap another entry's inputs or Y (LORA_ERR_ALIAS).  `descs` is a HOST
 * array of n entries, read during the call.  A problem with at least four
 * 128 x 128 output tiles per SM of the GPU runs as lora_fwd would; the
 * others share split-K launches (up to 40 problems per launch, longest
 * contraction first).  Results match lora_fwd within the forward tolerance
 * (the accumulation order may differ).
 */
typedef struct {
  const void* X;
  const void* W;
  const void* A;
  const void* B;
  void* Y;
  int64_t M;
  int64_t d_in;
  int64_t d_out;
} lora_fwd_desc_t;

lora_status_t lora_fwd_batched(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float alpha,
                               void* stream);

/*
 * Explicit scale.  Each of these is the entry point of the same name without
 * "_scaled", with the same arguments, rules and results, except that the
 * float `scale` takes the place of `alpha` and is used as s itself instead
 * of s = alpha / r.  rsLoRA is the case in point (unsloth fork commit log,
 * scripts/benchmarks/qwen3_flex_inference.py: under rsLoRA PEFT keeps
 * alpha / sqrt(r) in the module's scaling, and that value is what the layer
 * multiplies by); any other scale (0 gives the base layer alone) works the
 * same way.  A call with scale == alpha / r computed in fp32 gives the
 * results of the alpha form bit for bit.
 *   lora_fwd_scaled            <-> lora_fwd
 *   lora_fwd_save_scaled       <-> lora_fwd_save
 *   lora_fwd_batched_scaled    <-> lora_fwd_batched
 *   lora_bwd_scaled            <-> lora_bwd_ex (flags as there; 0 = lora_bwd)
 *   lora_bwd_grads_scaled      <-> lora_bwd_grads (lora_bwd_dx takes no scale)
 *   lora_merge_scaled          <-> lora_merge
 *   lora_merge_batched_scaled  <-> lora_merge_batched
 */
lora_status_t lora_fwd_scaled(const void* X, const void* W, const void* A, const void* B, void* Y,
                              int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                              void* stream);
lora_status_t lora_fwd_save_scaled(const void* X, const void* W, const void* A, const void* B, void* Y,
                                   int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream);
lora_status_t lora_fwd_batched_scaled(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float scale,
                                      void* stream);
lora_status_t lora_bwd_scaled(const void* X, const void* W, const void* A, const void* B,
                              const void* dY, void* dX, void* dA, void* dB,
                              int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                              void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);
lora_status_t lora_bwd_grads_scaled(const void* X, const void* A, const void* B, const void* dY, void* dA,
                                    void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                                    void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);
lora_status_t lora_merge_scaled(const void* W_src, const void* A, const void* B, void* W_dst,
                                int64_t d_out, int64_t d_in, int32_t r, float scale, void* stream);
lora_status_t lora_merge_batched_scaled(const lora_merge_desc_t* descs, int32_t n, int32_t r, float scale,
                                        void* stream);

/*
 * Restore: W_dst <- W_src, a bit copy of n_elems bf16 values (the pristine
 * copy is only read).
 */
lora_status_t lora_restore(const void* W_src, void* W_dst, int64_t n_elems, void* stream);

/*
 * Synchronizes the current device, returns LORA_ERR_TIMEOUT if any kernel
 * of this library gave up on a bounded wait since the last call (and clears
 * the flag), LORA_ERR_CUDA on a CUDA error, else LORA_OK.
 */
lora_status_t lora_get_device_status(void);

/*
 * Host-only validation (no GPU needed): checks pointers and sizes exactly as
 * the entry point for `op` would (op 0 = lora_fwd with ptrs {X,W,A,B,Y};
 * 1 = lora_bwd with {X,W,A,B,dY,dX,dA,dB,workspace}; 2 = lora_merge with
 * {W_src,A,B,W_dst}; M is ignored for op 2).  `workspace_bytes` is only
 * read for op 1.
 */
lora_status_t lora_check_args(int32_t op, const void* const* ptrs, int32_t n_ptrs,
                              int64_t M, int64_t d_in, int64_t d_out, int32_t r,
                              size_t workspace_bytes);

/*
 * Launch plan of a shape (a service of this library, not part of the method;
 * host only: no GPU needed, no device state read, nothing launched): the kernel configuration the library would choose on a
 * B200 with `sm_count` SMs, as the entry points choose it (including the
 * LORA_B200_* overrides in the environment).  For tests and tools; no
 * computation depends on these fields.  With M == 0 every field is zero.
 * Returns LORA_ERR_NULL for a NULL `out`, lora_fwd's SHAPE / RANK rules for
 * the sizes, and LORA_ERR_SHAPE for sm_count outside [2, 4096].
 */
typedef struct {
  int32_t fwd_kind;        /* 0 = tiled kernel (one output tile per CTA or CTA pair),
                              1 = split contraction (the CTAs of a cluster share a tile) */
  int32_t fwd_bn;          /* output tile width: 128 or 256; 224 = CTA pair with T folded into an N = 256 MMA */
  int32_t fwd_cg;          /* CTAs per tile (2 = CTA pair) */
  int32_t fwd_stages;      /* pipeline stages */
  int32_t fwd_run_l;       /* tiled: 0 = contiguous ranges, L = runs of L N tiles */
  int32_t fwd_num_m;       /* output tiles along M ... */
  int32_t fwd_num_n;       /* ... and along N */
  int32_t fwd_splits;      /* split contraction: CTAs per tile along K (tiled: 1) */
  uint32_t fwd_smem;       /* dynamic shared memory per CTA, bytes */
  int32_t bwd1_splits_dt;  /* backward launch 1: contraction splits of the dT job ... */
  int32_t bwd1_splits_t;   /* ... and of the T job (they share the launch) */
  int32_t bwd1_saved_splits; /* launch 1 with LORA_BWD_T_SAVED (dT alone) */
  uint32_t bwd1_smem;      /* launch 1: shared memory per CTA */
  int32_t bwd2_splits_db;  /* backward launch 2: splits of the dB job ... */
  int32_t bwd2_splits_da;  /* ... and of the dA job (they share the launch) */
  uint32_t bwd2_smem;
  int32_t dx_bn, dx_cg, dx_stages;  /* backward launch 3 (dX), tiled kernel */
  uint32_t dx_smem;
  uint64_t workspace_bytes; /* lora_bwd_workspace_size */
  int32_t fwd_seeded;      /* tiled: 1 = each cluster first runs fwd_run_l tiles of one M block
                              (computing its T for all), then the remaining tiles are dealt one at a
                              time; only with the exchange */
  int32_t fwd_tx;          /* tiled: 1 = clusters share the down-projection T (the exchange; with the
                              seeded schedule only) */
} lora_plan_t;

lora_status_t lora_plan(int64_t M, int64_t d_in, int64_t d_out, int32_t r, int32_t sm_count, lora_plan_t* out);

/*
 * Self-test of the bounded-wait machinery: launches one block that waits on
 * a barrier nothing will arrive on, with the given limit in nanoseconds
 * (clamped to [1e3, 1e9]).  Returns what lora_get_device_status() then
 * reports: LORA_ERR_TIMEOUT when the wait gave up as designed.
 */
lora_status_t lora_selftest_wait_timeout(int64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* LORA_B200_H */
