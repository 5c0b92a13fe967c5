/*
 * muon_b200.h -- C ABI of the B200 (sm_100a) Muon optimizer-step library.
 *
 * What the library computes (sources are the pages as titled, by section):
 *   - "きみはNanoGPT speedrunを知っているか？", section "Muonとは": Muon keeps a
 *     moving average of the gradient (momentum), approximately orthogonalises
 *     it by Newton-Schulz iteration and updates the parameters with the
 *     result; it applies to matrix parameters only.
 *   - neo-ai.one article, section "Muonが登場": the iteration drives the update
 *     toward a semi-orthogonal matrix and runs stably with bf16 operands.
 *   - "Training NanoGPT in 39.9 Seconds", section "ANVIL II와 가중치 평균": the
 *     two-momentum ANVIL variant (six polynomial applications, weight decay
 *     masked by agreement with the slow momentum) and the end-of-training EMA
 *     theta_bar <- beta theta_bar + (1 - beta) theta, readout blend 35/65.
 *   - "qlabs-eng/slowrun", section "仕組み": Muon with weight decay 1.6.
 *
 * Per matrix (R x C, r = min(R, C)) one Muon step is:
 *   M <- mu M + (1 - mu) G                         (moving-average momentum)
 *   U  = nesterov ? (1 - mu) G + mu M : M
 *   X  = U / (||U||_F + eps)          (U^T when R > C, so X is r x max(R, C))
 *   repeat ns_steps times, with that step's (a, b, c):
 *       A = X X^T ;  X <- a X + (b A + c A A) X
 *   O  = X (transposed back when R > C)
 *   theta <- theta (1 - lr wd) - lr max(1, R/C)^(1/2) O
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device (or managed) addresses on the current
 *     device; "host" marks host pointers. Matrices are row-major and
 *     contiguous; a bank of `count` matrices is [count][rows][cols].
 *   - The caller owns all memory, including the workspace. The library never
 *     allocates, frees or synchronises in the step calls; work is enqueued on
 *     `stream` (a cudaStream_t passed as void*, NULL = legacy default stream).
 *   - Arguments are validated on the host before anything is enqueued; a
 *     non-OK status means nothing was launched. MUON_OK from a step call
 *     means only that its work was enqueued. Faults found on the device (a
 *     bounded wait that ran out) are recorded in the workspace's status word
 *     and reported by muon_device_status, which synchronises: call it
 *     outside the hot loop, e.g. once every N steps or at a checkpoint.
 *   - The status word is sticky. In the step whose chain timed out the
 *     momenta have already advanced (the momentum pass runs first), but
 *     param, ema and O are left unchanged; every later step on that
 *     workspace leaves all of its buffers unchanged until the word is
 *     cleared (muon_device_status with clear != 0). Restore the momenta from
 *     a checkpoint before resuming if the failed step must not count.
 *   - One Newton-Schulz chain is a persistent launch whose CTA pairs wait on
 *     one another; its grid is capped at the pairs the device can hold at
 *     once. Kernels of other streams that hold SMs only delay a chain, and
 *     chains on streams of equal priority are dispatched in launch order and
 *     serialise. A chain on a higher-priority stream can take SMs that an
 *     earlier chain still needs; both then end with MUON_ERR_TIMEOUT (the
 *     waits are bounded). Run one chain at a time per device, or give the
 *     streams that carry steps the same priority.
 *   - Every device pointer must be 16-byte aligned. param, momentum,
 *     momentum_slow and ema are updated in place and must not overlap one
 *     another, in the same bank or in another bank of the call (checked:
 *     MUON_ERR_ALIAS), nor the workspace (not checked); grad is read only.
 *   - Size limits (MUON_ERR_SHAPE beyond them): rows and cols, rounded up
 *     to 256, below 2^24; per bank, count times the rounded rows below 2^31,
 *     and below 2^30 its 256 x 256 output tiles and its 8192-element blocks;
 *     over all banks of a call, the chain's tiles (every phase, times
 *     ns_steps) and the elementwise blocks below 2^31: the kernels index
 *     them with 32-bit integers.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 2
#define MUON_MAX_NS_STEPS 16
#define MUON_MAX_BANKS 8

typedef enum {
  MUON_OK = 0,
  MUON_ERR_NULL = 1,        /* a required pointer is NULL                     */
  MUON_ERR_SHAPE = 2,       /* count/rows/cols < 1 or too large, nbanks range */
  MUON_ERR_DTYPE = 3,       /* unsupported dtype code                         */
  MUON_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned        */
  MUON_ERR_HPARAM = 5,      /* ns_steps outside 1..16, non-finite or out-of-range scalar */
  MUON_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than muon_workspace_size */
  MUON_ERR_CUDA = 7,        /* a CUDA runtime call failed (launch, attribute) */
  MUON_ERR_TIMEOUT = 8,     /* a bounded device-side wait ran out             */
  MUON_ERR_ALIAS = 9,       /* in-place buffers overlap                       */
  MUON_ERR_BOUNDS = 10      /* debug build only: an index outside its buffer
                               (the access was skipped; results invalid)      */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype;

/* One bank of `count` same-shape rows x cols matrices. */
typedef struct {
  int64_t count, rows, cols;
  void* param;              /* device, [count][rows][cols], param_dtype, in/out     */
  int32_t param_dtype;      /* MUON_F32 or MUON_BF16                                */
  int32_t grad_dtype;       /* MUON_F32 or MUON_BF16                                */
  const void* grad;         /* device, [count][rows][cols], grad_dtype, read only   */
  float* momentum;          /* device fp32 [count][rows][cols]: M (Muon) or M_fast (ANVIL), in/out */
  float* momentum_slow;     /* device fp32, ANVIL's slow momentum, in/out; NULL for Muon */
  float* ema;               /* device fp32 EMA of param, in/out; NULL = no EMA       */
} muon_bank;

/* Hyper-parameters (host struct, copied by value at each call). */
typedef struct {
  float lr;                 /* learning rate (> 0 not required; finite)              */
  float mu;                 /* Muon momentum, 0 <= mu < 1                             */
  float weight_decay;       /* decoupled (Muon) or cautious (ANVIL) decay, >= 0       */
  float eps;                /* added to ||U||_F before dividing, >= 0 (1e-7 usual)    */
  int32_t nesterov;         /* Muon: 1 = U = (1-mu) G + mu M, 0 = U = M               */
  int32_t ns_steps;         /* 1..MUON_MAX_NS_STEPS                                   */
  float coeffs[3 * MUON_MAX_NS_STEPS]; /* (a, b, c) of step i at coeffs[3i..3i+2]     */
  float ema_beta;           /* 0 <= beta < 1; used when a bank has ema != NULL        */
  float beta_fast;          /* ANVIL fast-momentum beta, 0 <= beta < 1                */
  float beta_slow;          /* ANVIL slow-momentum beta, 0 <= beta < 1                */
  int32_t sgd_momentum;     /* Muon only. 0: moving average M <- mu M + (1-mu) G
                             * (Nesterov U = (1-mu) G + mu M); 1: SGD form
                             * M <- mu M + G (Nesterov U = G + mu M). From zero state
                             * the SGD buffer is the moving average / (1 - mu), so
                             * both forms give the same update O.               */
} muon_hparams;

/* ABI version of the loaded library (MUON_ABI_VERSION). */
int32_t muon_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* muon_status_string(muon_status s);

/* Bytes of device workspace that muon_step / anvil_step / muon_orthogonalize
 * need for these banks (host-only computation; 0 if the banks are invalid).
 * Zero-fill a new workspace once before its first use (its first bytes hold
 * the device status word); its contents need no other initialisation. The
 * workspace holds the Newton-Schulz iterate as a bf16 hi/lo pair (two hi
 * buffers), the bf16 Gram matrix A and polynomial B, and per-matrix norms. */
size_t muon_workspace_size(const muon_bank* banks, int32_t nbanks);

/* One Muon step for `nbanks` banks (host array) -- the sequence at the top of
 * this file ("Muonとは", "Muonが登場"). Uses param, grad, momentum, ema (if not
 * NULL: updated after the parameter write with the stored parameter value)
 * and hp.lr, mu, weight_decay, eps, nesterov, ns_steps, coeffs, ema_beta.
 * ws: device workspace of ws_bytes >= muon_workspace_size(banks, nbanks). */
muon_status muon_step(const muon_bank* banks, int32_t nbanks, const muon_hparams* hp,
                      void* ws, size_t ws_bytes, void* stream);

/* One ANVIL-style step ("ANVIL II와 가중치 평균"): M_fast and M_slow are moving
 * averages of G with hp.beta_fast / hp.beta_slow; the fast one is normalised
 * and put through the ns_steps polynomial applications (no Nesterov); the
 * decay is applied only where O * M_slow > 0:
 *   theta <- theta - lr wd [O M_slow > 0] theta - lr max(1,R/C)^(1/2) O.
 * momentum = M_fast, momentum_slow = M_slow (both required); optional EMA as
 * in muon_step. */
muon_status anvil_step(const muon_bank* banks, int32_t nbanks, const muon_hparams* hp,
                       void* ws, size_t ws_bytes, void* stream);

/* The orthogonalisation alone: out = NS(in / (||in||_F + eps)) per matrix
 * (transpose rule as above). in: device [count][rows][cols] (in_dtype);
 * out: device, same shape, out_dtype. Uses hp.eps, ns_steps, coeffs only.
 * ws sized by muon_workspace_size for a bank of that shape. */
muon_status muon_orthogonalize(const void* in, int32_t in_dtype, void* out, int32_t out_dtype,
                               int64_t count, int64_t rows, int64_t cols,
                               const muon_hparams* hp, void* ws, size_t ws_bytes, void* stream);

/* muon_orthogonalize without a caller workspace. The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves, for example a plug-in inside a host application
 * that owns every device allocation, or a latency-critical loop where a
 * cudaMalloc (which may synchronise the whole device) is not allowed. Its
 * scratch memory is one array of MUON_STATIC_SCRATCH_BYTES in the library's
 * own device memory, reserved on every GPU that loads the library until the
 * process exits. Arguments and results are those of muon_orthogonalize
 * (inputs and outputs still belong to the caller).
 *   - A bank whose muon_workspace_size exceeds MUON_STATIC_SCRATCH_BYTES is
 *     rejected with MUON_ERR_WORKSPACE before anything is launched (32 MiB
 *     holds e.g. one 768 x 3072 or two 1024 x 1024 matrices).
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     each call clears the part that must start at zero. Calls whose work
 *     overlaps on the GPU (other streams, other host threads) race on it.
 *   - The device status word used by bounded waits lives in the array too and
 *     is cleared at the start of every call, so a timeout here is not visible
 *     to muon_device_status; use muon_orthogonalize to observe it.
 * Calls no cudaMalloc, cudaFree or other allocating routine. */
#define MUON_STATIC_SCRATCH_BYTES (32u << 20)
muon_status muon_orthogonalize_static(const void* in, int32_t in_dtype, void* out,
                                      int32_t out_dtype, int64_t count, int64_t rows,
                                      int64_t cols, const muon_hparams* hp, void* stream);

/* EMA of the parameters ("ANVIL II와 가중치 평균", averaging equation):
 * ema <- beta ema + (1 - beta) param, for every bank with ema != NULL.
 * 0 <= beta < 1. Banks whose ema is NULL are skipped. */
muon_status ema_update(const muon_bank* banks, int32_t nbanks, float beta, void* stream);

/* Readout blend ("ANVIL II와 가중치 평균": 35 % final, 65 % average):
 * out[i] = w_final theta[i] + (1 - w_final) ema[i], i < n.
 * theta: device (theta_dtype); ema: device fp32; out: device (out_dtype). */
muon_status readout_blend(const void* theta, int32_t theta_dtype, const float* ema,
                          void* out, int32_t out_dtype, int64_t n, float w_final,
                          void* stream);

/* Synchronises `stream`, then reads the workspace's device status word:
 * MUON_OK, or MUON_ERR_TIMEOUT if a bounded wait inside a kernel ran out
 * since the word was last cleared. clear != 0 resets it to MUON_OK. This
 * call blocks the host and is not meant for the hot loop. */
muon_status muon_device_status(void* ws, size_t ws_bytes, void* stream, int32_t clear);

/* Instrumentation hook, process-wide. The next muon_step, anvil_step or
 * muon_orthogonalize call records `before_ns` on its stream right before its
 * first Newton-Schulz launch and `after_ns` right after its last one, then
 * forgets both. Both are cudaEvent_t handles passed as void* (created by the
 * caller with timing enabled); NULL, NULL clears a pending pair. */
muon_status muon_set_ns_events(void* before_ns, void* after_ns);

/* Host only, no GPU needed: the Newton-Schulz chain's tile list for banks of
 * the given shapes and ns_steps, as the kernel decodes it (for tests and
 * tooling). shapes: host array of 3 * nbanks values, (count, rows, cols) of
 * bank b at shapes[3b..3b+2], validated like a step's banks. tiles: host array
 * owned by the caller, or NULL to only count. Tiles are listed step by step, phase by
 * phase (Gram, Reduce, Poly, Apply), bank by bank, matrix by matrix. If
 * tiles_cap >= 13 * (number of tiles), tiles[13t..13t+12] = (step, phase
 * (0 Gram, 1 Poly, 2 Apply, 3 Reduce), bank, matrix, first output row, first
 * output column, first 64-deep K block, K blocks, left operand map slot, left
 * operand base row, right operand map slot, right operand base row, 1 if the
 * right operand is the left one and is not loaded) of tile t. Returns the
 * number of tiles, or minus a muon_status on invalid input. */
int64_t muon_chain_plan(const int64_t* shapes, int32_t nbanks, int32_t ns_steps, int32_t* tiles,
                        int64_t tiles_cap);

/* Test hook, process-wide. wait_limit_seconds bounds every device-side wait
 * (default 2 s; values <= 0 restore the default). fault_mode 0 = normal;
 * 1 = the Newton-Schulz kernel's producer withholds the first operand stage of
 * block 0's first tile, so the consumer's bounded wait runs out and the call
 * reports MUON_ERR_TIMEOUT through muon_device_status (results invalid). */
muon_status muon_set_debug(int32_t fault_mode, double wait_limit_seconds);

#ifdef __cplusplus
}
#endif
#endif /* MUON_B200_H */
