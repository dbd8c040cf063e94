/*
 * vsa.h -- C ABI of libvsa.so: the forward pass of VSA-style cube-based
 * hierarchical sparse attention on one NVIDIA B200 (sm_100a).
 *
 * The method (sources are web pages about it, cited by title and section):
 *   "Faster Video Diffusion with Trainable Sparse Attention", "Approach":
 *     mean-pool tokens into 4x4x4 cubes, run a coarse cube-to-cube dense
 *     attention that outputs a coarse context and selects the top-K critical
 *     cubes per query cube, run block-sparse token-level fine attention only
 *     over the selected cubes, and combine both outputs through gates; each
 *     cube maps to one GPU tile.
 *   same page, "Limitations": the cube size is fixed at (4,4,4), so T, H and
 *     W must be multiples of 4.
 *   "Improving Video Sparse Attention with Fine-grained Router and Sparse
 *     Rebasing", "Abstract (arXiv)": each query may attend to a variable
 *     number of key-value blocks (read here as a top-p rule, see topk/top_p).
 *
 * Conventions used by every entry point
 *   Tensors are dense, row-major, on the current CUDA device:
 *     q, k, v, out     [B, heads, N, D]   bfloat16   (N = T*H*W, raster order
 *                                          n = (t*H + h)*W + w)
 *     gate_c, gate_f   [B, heads, N]      float32    (one scalar per token and
 *                                          head; used as given)
 *     idx              [B, heads, C, Kcap] int32     (C = N/64; selected KV
 *                                          cube ids per query cube, ascending,
 *                                          padded with -1)
 *     cnt              [B, heads, C]      int32      (number of valid ids)
 *   Cube numbering: cube c = ((t/4)*(H/4) + h/4)*(W/4) + w/4; the 64 tokens
 *   of a cube are ordered ((t%4)*4 + h%4)*4 + w%4.
 *   Scores use scale 1/sqrt(D). Ties in the coarse score go to the lower
 *   cube id.
 *   All pointers are owned by the caller; the library never frees them.
 *   Every pointer argument must be 16-byte aligned.
 *   Calls only enqueue work on `stream` (a cudaStream_t passed as void*; NULL
 *   is the legacy default stream) and return without synchronising, except
 *   vsa_check. Host-side argument errors are reported synchronously and no
 *   work is enqueued. A failed kernel launch returns VSA_ERR_CUDA. Errors
 *   detected on the device (a bounded wait that gave up) are recorded in the
 *   plan's workspace and returned by the next vsa_check.
 *   Threads may share a plan: its calls take a per-plan lock for their
 *   host-side work (tensor-map encoding, launches). The plan has one
 *   workspace, though, so the device work of two calls on different streams
 *   without ordering between them races on it: order such calls (one
 *   stream, or events).
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1, /* null pointer, bad count, bad mode parameters   */
  VSA_ERR_SHAPE = 2,       /* T, H or W not a multiple of 4; B or heads < 1  */
  VSA_ERR_UNSUPPORTED = 3, /* D not in {64, 128}; C or Kcap beyond limits    */
  VSA_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned               */
  VSA_ERR_CUDA = 5,        /* a CUDA call or kernel launch failed            */
  VSA_ERR_TIMEOUT = 6,     /* a device-side wait gave up (see vsa_check)     */
  VSA_ERR_DEVICE = 7       /* the device is not an sm_100 part               */
} vsa_status;

/* Problem description.
 *   topk > 0 : fixed top-K mode, 1 <= topk <= C, Kcap = topk.
 *   topk == 0: top-p mode. For query cube i, rank the KV cubes by coarse
 *              score and keep the shortest prefix whose coarse softmax mass
 *              reaches top_p (inclusive; all C if none does), then clamp the
 *              count to [kmin, kmax]. 0 < top_p <= 1, 1 <= kmin <= kmax <= C,
 *              Kcap = kmax.
 * Limits: D in {64, 128}; C <= 4096; Kcap <= C. */
typedef struct {
  int B, heads, T, H, W, D;
  int topk;
  float top_p;
  int kmin, kmax;
} vsa_config;

typedef struct vsa_plan_s* vsa_plan_t;

/* Byte offsets of the plan's workspace regions (for inspection by tests and
 * tools). All are relative to the workspace base passed to vsa_plan. */
typedef struct {
  size_t q_cube, k_cube, v_cube; /* [B*heads, C, 64, D] bf16, cube-major copies
                                    (q's only with vsa_set_cube_major_copies)     */
  size_t q_pool, k_pool, v_pool; /* [B*heads, C, D] fp32 cube means               */
  size_t o_coarse;               /* [B*heads, C, D] fp32 coarse output            */
  size_t s_coarse;               /* [B*heads, C, C] fp32 coarse scores             */
  size_t pool_split;             /* [3 (q, k, v), 3, B*heads, C, D] bf16: each cube
                                    mean as three bf16 terms hi + mid + lo        */
  size_t p_split;                /* [3, B*heads, C, Cp] bf16: the coarse softmax
                                    probabilities as three bf16 terms, Cp = C
                                    rounded up to a multiple of 8 (zero padded)   */
  size_t cnt;                    /* [B*heads, C] int32 counts used by the fine step */
  size_t order;                  /* [B*heads*C] int32 work order of the fine step
                                    when counts vary (each head's query cubes
                                    longest first)                              */
  size_t err;                    /* int32 device error word                        */
  size_t total;                  /* == vsa_workspace_bytes                          */
} vsa_workspace_layout_t;

/* Workspace size in bytes for cfg, or 0 if cfg is invalid. */
size_t vsa_workspace_bytes(const vsa_config* cfg);

/* Fills *layout for cfg. Returns VSA_OK or the validation error of cfg. */
vsa_status vsa_workspace_layout(const vsa_config* cfg, vsa_workspace_layout_t* layout);

/* Validates cfg and builds a plan over a caller-provided device workspace of
 * at least vsa_workspace_bytes(cfg) bytes (256-byte aligned). The plan keeps
 * the tensor-map descriptors of the workspace; it allocates host memory only.
 * The workspace must stay valid until vsa_plan_destroy. */
vsa_status vsa_plan(vsa_plan_t* out, const vsa_config* cfg, void* workspace, size_t ws_bytes);

/* Whole forward pass: cube gather + mean pool, coarse attention + selection,
 * block-sparse fine attention + gated combine.
 *   out: [B,heads,N,D] bf16; idx: [B,heads,C,Kcap] int32 (written);
 *   cnt: [B,heads,C] int32 (written) or NULL. */
vsa_status vsa_run(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                   const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* stream);

/* Forward pass on a caller-supplied selection (the selection step is not run).
 *   idx_in: [B,heads,C,Kcap] ascending cube ids; cnt_in: [B,heads,C] or NULL
 *   (NULL means every row holds Kcap ids).
 *   out: gated output (bf16, may be NULL);
 *   out_coarse: [B,heads,C,D] fp32 coarse output (may be NULL);
 *   out_fine:   [B,heads,N,D] fp32 fine-attention output before gating
 *               (may be NULL). */
vsa_status vsa_run_fixed_idx(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                             const float* gate_f, const int32_t* idx_in, const int32_t* cnt_in, void* out,
                             float* out_coarse, float* out_fine, void* stream);

/* Training forward pass: vsa_run, and it also saves what vsa_run_backward
 * needs ("Faster Video Diffusion with Trainable Sparse Attention",
 * "Approach": the hierarchy is trained end to end; "VSA: Faster Video
 * Diffusion with Trainable Sparse Attention", "Abstract (arXiv)": a single
 * differentiable kernel).
 *   o_fine: [B,heads,N,D] fp32, written: the fine-attention output before
 *           gating (raster order). fp32 because the backward pass forms
 *           delta_n = dO_n . O_n from it: with O rounded to bf16 the error of
 *           delta, multiplied by the softmax-weighted mean key in dq, can
 *           exceed dq itself where attention is spread over similar keys.
 *   lse:    [B,heads,N] fp32, written: per token n, the natural log of its
 *           fine softmax denominator, log(sum_m exp(q_n . k_m / sqrt(D))) over
 *           the tokens m of its query cube's selected cubes (raster order).
 *   out, idx, cnt as in vsa_run (cnt may be NULL). */
vsa_status vsa_run_train(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                         const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* o_fine, float* lse,
                         void* stream);

/* Bytes of device workspace vsa_run_backward needs for cfg (0 if cfg is
 * invalid): dO in cube-major order, per-token statistics, the coarse
 * backward's C x C products and the transposed selection lists. */
size_t vsa_backward_workspace_bytes(const vsa_config* cfg);

/* Backward pass of the forward pass with the selection held fixed (an index
 * choice has no gradient; the pages give no gradient formulas, so these are
 * the chain rule of the forward computation):
 *   dgate_c[n] = dout_n . Oc[cube(n)]          dgate_f[n] = dout_n . Of_n
 *   fine (per query cube i over the tokens of its selected cubes, with
 *   dOf = gate_f dout, P = exp(q k^T/sqrt(D) - lse), delta_n = dOf_n . Of_n):
 *     dS = P o (dOf v^T - delta); dq = dS k / sqrt(D); dk = dS^T q / sqrt(D);
 *     dv = P^T dOf, the key and value terms summed over every query cube
 *     that selected the cube;
 *   coarse (dense over the pooled tokens, dOc[c] = sum over cube c's tokens
 *   of gate_c dout): the attention gradient of the means, handed to every
 *   token of a cube with weight 1/64 (the mean's derivative).
 * Inputs: q, k, v, gate_c, gate_f as given to vsa_run_train; idx, cnt the
 *   selection it returned (cnt may be NULL in top-K mode; every row must be
 *   strictly ascending, ids in [0, C), counts in [1, Kcap]); o_fine and lse
 *   the tensors it saved; dout [B,heads,N,D] bf16, the gradient of out.
 * Outputs (written): dq, dk, dv [B,heads,N,D] bf16; dgate_c, dgate_f
 *   [B,heads,N] fp32.
 * bwd_workspace: device memory of at least vsa_backward_workspace_bytes(cfg)
 *   bytes, 256-byte aligned, owned by the caller. The call also recomputes
 *   the gather and the coarse stage into the plan's workspace (so the plan's
 *   workspace contents of an earlier forward call are overwritten).
 * Two kernels compute the fine gradients without atomics (query-major dq,
 * KV-major dk and dv), so the results are deterministic. A malformed
 * selection (id out of range, a row not strictly ascending, a count outside
 * [1, Kcap]) is never used as an address; it is reported by vsa_check as
 * VSA_ERR_INVALID_ARG and its gradients are then unspecified. */
vsa_status vsa_run_backward(vsa_plan_t plan, void* bwd_workspace, size_t bwd_bytes, const void* q, const void* k,
                            const void* v, const float* gate_c, const float* gate_f, const int32_t* idx,
                            const int32_t* cnt, const void* o_fine, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, float* dgate_c, float* dgate_f, void* stream);

/* Forward pass on HOST buffers: copies the inputs to the device, runs the
 * forward pass (as vsa_run) and copies the results back, all enqueued on
 * `stream`. The pages describing the method have no counterpart of this
 * entry point; it is the path for callers whose tensors live in host memory.
 * The work is split by (batch, head): the copy of slice i+1 to the device
 * and of slice i-1 back to the host run on two library streams while slice
 * i is computed on `stream`, so the copies overlap the computation (and
 * each other) when the host buffers are pinned (page-locked); pageable
 * buffers work too, without overlap.
 *   q, k, v: [B,heads,N,D] bf16 host; gate_c, gate_f: [B,heads,N] fp32 host;
 *   out: [B,heads,N,D] bf16 host (written); idx: [B,heads,C,Kcap] int32 host
 *   (written); cnt: [B,heads,C] int32 host (written) or NULL.
 * The host results are complete once `stream` has reached the end of the
 * call's work (synchronise it before reading them). The first call on a plan
 * allocates device copies of the inputs and results (B*heads*(5*N*D*2 +
 * 2*N*4 + C*Kcap*4 + C*4) bytes, rounded up), a workspace for one
 * (batch, head) slice and two streams; later calls allocate nothing and the
 * plan releases them in vsa_plan_destroy. Device-side errors are reported by
 * vsa_check(plan). Returns VSA_ERR_INVALID_ARG for a NULL argument (other
 * than cnt) and VSA_ERR_CUDA if a copy, an allocation or a launch fails. */
vsa_status vsa_run_host(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                        const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* stream);

/* One-call form. Keeps a library-owned plan and workspace per distinct
 * configuration and device (the first call for a configuration allocates
 * device memory with cudaMalloc; later calls allocate nothing). At most 16
 * configurations are kept, for the life of the process; a call with a 17th
 * returns VSA_ERR_UNSUPPORTED (use vsa_plan for more). topk > 0 selects top-K;
 * topk == 0 selects top-p with kmin = 4 and kmax = min(128, C).
 * Calls with the same configuration on the same device share one cached
 * plan and workspace: calls whose device work overlaps (different streams
 * without ordering, or host threads that do not order their streams) race on
 * that workspace, so serialise them. Device-side errors (a bounded wait that
 * gave up) are not reported by this form, which has no plan to pass to
 * vsa_check; use vsa_plan / vsa_run where they must be seen. */
vsa_status vsa_forward(const void* q, const void* k, const void* v, const float* gate_c, const float* gate_f,
                       int B, int heads, int T, int H, int W, int D, int topk, float top_p, void* out, int32_t* idx,
                       void* stream);

/* Forward pass for callers that cannot allocate memory: for example code
 * running under a strict memory budget, inside a custom allocator that must
 * own every device byte, or in a real-time loop where cudaMalloc (which may
 * synchronise the device) is not allowed. It takes the same arguments and
 * returns the same results as vsa_forward, but allocates nothing -- no
 * cudaMalloc, no host heap: its workspace is one fixed device array of
 * VSA_NOALLOC_SCRATCH_BYTES inside libvsa.so, which every GPU that loads
 * the library holds until the process exits.
 * The pages describing the method have no counterpart of this entry point.
 *   - Configurations whose workspace exceeds VSA_NOALLOC_SCRATCH_BYTES are
 *     rejected with VSA_ERR_UNSUPPORTED before anything is enqueued. The
 *     workspace here is vsa_workspace_bytes(cfg) less the q_cube region,
 *     which this entry point never writes: e.g. up to 6 heads of D = 128 at
 *     16,384 tokens (58.1 MiB) fit, 7 do not.
 *   - The first call on each device looks up the device address of the
 *     array (cudaGetSymbolAddress); make that first call before any stream
 *     capture starts.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (different streams, or different host threads, without ordering
 *     between them) race on it. Serialise them, e.g. on one stream.
 *   - The array keeps the previous call's contents; the call clears the
 *     part that must start at zero (the device error word) itself.
 *   - Device-side errors of this entry point are not reported (there is no
 *     plan to query with vsa_check). */
#define VSA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
vsa_status vsa_forward_noalloc(const void* q, const void* k, const void* v, const float* gate_c,
                               const float* gate_f, int B, int heads, int T, int H, int W, int D, int topk,
                               float top_p, void* out, int32_t* idx, void* stream);

/* Synchronises the stream the plan last ran on, then reports (and clears) the
 * device error word: VSA_OK; VSA_ERR_TIMEOUT if a device wait gave up;
 * VSA_ERR_INVALID_ARG if vsa_run_fixed_idx was given a cube id outside [0, C)
 * or a count outside [1, Kcap] (the kernel substituted cube 0 / clamped the
 * count instead of reading out of bounds); VSA_ERR_CUDA if the stream
 * reported an error. */
vsa_status vsa_check(vsa_plan_t plan);

/* Releases the plan (host memory only; the workspace stays the caller's). */
void vsa_plan_destroy(vsa_plan_t plan);

/* Static, human-readable name of a status code. */
const char* vsa_status_string(vsa_status s);

/* Device-side wait limit in nanoseconds used by later launches of this plan
 * (default 1e9, minimum 1e5). Every wait of a kernel on an mbarrier gives
 * up after this long, records VSA_ERR_TIMEOUT in the workspace error word,
 * drains the copies and tensor-core operations it already issued, and
 * returns. */
vsa_status vsa_set_wait_limit_ns(vsa_plan_t plan, uint64_t limit_ns);

/* Test hook for the timeout path. When `on` is nonzero, the fine-attention
 * kernel's tensor-core issuer first waits on a barrier that nothing ever
 * signals, so that wait runs out after the plan's wait limit and the run
 * ends with VSA_ERR_TIMEOUT (reported by vsa_check) instead of hanging. */
vsa_status vsa_set_debug_stall(vsa_plan_t plan, int on);

/* Inspection switch for the gather step (raster -> cube-major reorder;
 * "Faster Video Diffusion with Trainable Sparse Attention", "Approach": one
 * cube of 4 x 4 x 4 tokens is one tile). Every run writes the cube-major
 * copies of k and v (regions k_cube, v_cube), which the fine-attention kernel
 * streams; it reads q straight from the raster tensor (16-byte copies of each
 * query cube's token rows), so q's copy is not needed. When `on` is nonzero, later runs of this plan also
 * write q's copy into region q_cube (one extra write of q); off by default. */
vsa_status vsa_set_cube_major_copies(vsa_plan_t plan, int on);

/* Stage timing for benchmarks. When `on` is positive, later runs of this plan
 * record CUDA events on the run's stream around its three stages: gather +
 * pool, coarse attention + selection, fine attention + combine; the events of
 * the last `on` runs are kept (at most 4096; created here), and likewise the
 * four stages of vsa_run_backward calls. 0 switches timing off. Every call
 * restarts the counts of recorded runs. */
vsa_status vsa_set_stage_timing(vsa_plan_t plan, int on);

/* Waits for the events of the last timed run and writes the device time of
 * its stages in milliseconds to ms[0] (gather + pool), ms[1] (coarse),
 * ms[2] (fine). VSA_ERR_INVALID_ARG if timing is off or nothing ran yet. */
vsa_status vsa_stage_times(vsa_plan_t plan, float* ms);

/* The stage times of the last min(max_runs, runs kept) timed runs, oldest
 * first: ms[3 i + s] for run i and stage s (as in vsa_stage_times); the
 * number of runs written goes to *n_runs. Waits for the last run's events. */
vsa_status vsa_stage_times_history(vsa_plan_t plan, float* ms, int max_runs, int* n_runs);

/* Waits for the events of the last timed vsa_run_backward and writes the
 * device time of its stages in milliseconds: ms[0] gather + coarse forward
 * (recomputed), ms[1] per-token preparation + transposed lists + coarse
 * backward, ms[2] fine dq, ms[3] fine dk / dv. VSA_ERR_INVALID_ARG if timing
 * is off or no backward ran since it was switched on. */
vsa_status vsa_backward_stage_times(vsa_plan_t plan, float* ms);

/* The backward stage times of the last min(max_runs, runs kept) timed
 * vsa_run_backward calls, oldest first: ms[4 i + s] for call i and stage s
 * (as in vsa_backward_stage_times); the count goes to *n_runs. */
vsa_status vsa_backward_stage_times_history(vsa_plan_t plan, float* ms, int max_runs, int* n_runs);

/* Number of kernel launches one vsa_run / vsa_run_fixed_idx call makes in
 * top-K mode (5). With variable counts (top-p, or vsa_run_fixed_idx given
 * counts) one more kernel orders the fine step's work longest first. */
int vsa_kernels_per_run(void);

/* Measurement hook (not a step of the method; the pages have no counterpart):
 * enqueues one kernel that reads the first floor(bytes / 16384) * 16384
 * bytes of the device buffer `buf` `passes` times, in 16 KB untiled bulk
 * copies into shared memory (the TMA engine, as the fine-attention kernel
 * loads its K/V tiles), two CTAs per SM. Time it with events on `stream`;
 * with a buffer that fits in L2 (and a first pass to bring it there) the
 * rate is the L2 -> SM bandwidth of such copies. Nothing is written except
 * *status (a device int the caller zeroes): bit 0 is set if a bounded wait
 * gave up. buf and status must be 16-byte aligned; bytes >= 16384. */
vsa_status vsa_measure_l2_read(const void* buf, size_t bytes, int passes, int* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* VSA_H_ */
