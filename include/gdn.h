/*
 * gdn.h -- C ABI of libgdn.so: chunked-prefill forward and backward of the
 * Gated Delta Network (GDN) linear-attention layer on NVIDIA B200 (sm_100a).
 *
 * The operation.  The FlashQLA pages (news.hamidun.com "Qwen FlashQLA ... Hopper",
 * section "What is FlashQLA"; dothoosh.com FlashQLA article, opening paragraphs)
 * describe kernels for the forward and backward passes of GDN in chunked-prefill
 * mode.  Per sequence and value head the layer is the gated delta rule
 *
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 *
 * with an optional initial state S_0 and the final state S_T returned, so that a
 * long prompt can be fed as consecutive calls, each call's S_T becoming the
 * next call's S_0 (news.hamidun.com page, "Chunked Prefill" scenario).
 *
 * State layout.  Every state array stores H = S^T, i.e. [dk][dv] row-major per
 * (sequence, value head), so that o_t = H^T q_t.
 *
 * Heads.  q/k have Hk heads and v has Hv heads, Hv a multiple of Hk; value
 * head h reads q/k head h / (Hv / Hk) (contiguous groups).  beta and g are
 * per (token, value head).  No 1/sqrt(dk) scale is applied to q.
 *
 * Tensors (all device memory unless noted, contiguous, row-major):
 *   q, k   [B, T, Hk, dk]  dtype        v, o     [B, T, Hv, dv]  dtype
 *   beta, g [B, T, Hv]     fp32         S0, ST   [N, Hv, dk, dv]  fp32
 * dtype is fp32 or bf16 (GDN_F32 / GDN_BF16).  g is the raw per-token log decay
 * (not a cumulative sum); it must be finite.
 * Variable-length batches: pass cu_seqlens (int32 [N+1], device) together with
 * its host copy cu_seqlens_host; then B must be 1, T is the total token count
 * and sequence n owns tokens [cu[n], cu[n+1]).  Without cu_seqlens, N = B.
 *
 * Ownership and ordering.  The caller owns every buffer, the workspace
 * included; the library allocates no memory and keeps no state between calls.
 * Every entry point is asynchronous on the given stream: it enqueues kernels
 * and returns without synchronising, so buffers must stay valid until the
 * stream reaches that point.  Calls on different streams may run from
 * different host threads.  Inputs are never written.
 *
 * Errors.  Arguments are checked on the host before anything is launched;
 * GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED / GDN_ERR_WORKSPACE then mean that
 * nothing was enqueued.  GDN_ERR_CUDA means a launch failed (the CUDA error is
 * not cleared).  Device-side problems (a bounded wait that expired) are written
 * as a gdn_status value into *dev_status when dev_status is non-NULL; the
 * caller reads it after its own synchronisation.  Kernels never trap.  Nothing
 * throws across this interface.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#define GDN_ABI_VERSION 1u
#define GDN_CHUNK 64 /* tokens per chunk of the chunked algorithm */

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* NULL / inconsistent / misaligned argument      */
    GDN_ERR_UNSUPPORTED = 2, /* well-formed but outside what is implemented    */
    GDN_ERR_WORKSPACE = 3,   /* workspace NULL, too small or not 256-B aligned */
    GDN_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed           */
    GDN_ERR_TIMEOUT = 5,     /* device: a bounded wait expired                 */
    GDN_ERR_DEVICE = 6,      /* device: an internal consistency check failed   */
    GDN_ERR_TOO_LARGE = 7    /* gdn_chunk_fwd_noalloc: problem exceeds its scratch */
} gdn_status;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* flags (bitwise or); 0 selects the defaults */
#define GDN_FLAG_SPLIT_OFF (1u << 0)   /* never split one sequence across SMs      */
#define GDN_FLAG_SPLIT_FORCE (1u << 1) /* split every sequence into short segments */
#define GDN_FLAG_PORTABLE (1u << 2)    /* test aid: run a shape that the tensor-core
                                          kernels cover on the CUDA-core kernels instead
                                          (fp32 arithmetic), to cross-check the two; not
                                          a second backend for production use          */
#define GDN_FLAG_GATE_LOGITS (1u << 3) /* raw gates: beta holds logits b, beta =
                                          sigmoid(b); g holds pre-activations a, g =
                                          -softplus(a) = -log(1 + e^a); the backward's
                                          dbeta and dg are then gradients with respect to
                                          b and a.  Forward, backward and decode step.  */
#define GDN_FLAG_QK_L2NORM (1u << 4)   /* raw q and k: each (token, head) row is
                                          normalised over the head dimension,
                                          x / max(|x|_2, 1e-6) in fp32, before use; dq
                                          and dk are then gradients with respect to the
                                          raw rows.  Forward, backward and decode step. */

/* Arguments of the forward.  struct_size = sizeof(gdn_fwd_args),
 * abi_version = GDN_ABI_VERSION. */
typedef struct gdn_fwd_args {
    uint32_t struct_size;
    uint32_t abi_version;
    int32_t dtype;    /* gdn_dtype of q, k, v and o                          */
    int32_t B, T;     /* batch and tokens per sequence (total tokens if varlen) */
    int32_t Hk, Hv;   /* q/k heads, value heads (Hv % Hk == 0)                 */
    int32_t dk, dv;   /* head dims, 1..128 (tensor-core path: 128 x 128 bf16)  */
    int32_t num_seqs; /* N when cu_seqlens != NULL, else ignored (N = B)       */
    uint32_t flags;
    const void* q;
    const void* k;
    const void* v;
    const float* beta;
    const float* g;
    const int32_t* cu_seqlens;      /* device [N+1] or NULL                      */
    const int32_t* cu_seqlens_host; /* host copy, required with cu_seqlens       */
    const float* S0;                /* [N,Hv,dk,dv] or NULL (zero initial state) */
    void* o;                        /* out [B,T,Hv,dv], dtype                    */
    float* ST;                      /* out [N,Hv,dk,dv] or NULL (not written);
                                       must not overlap S0 (GDN_ERR_INVALID_ARG):
                                       a split sequence may read S0 after S_T of
                                       the same sequence was written              */
    int32_t* dev_status;            /* device int32 or NULL                      */
} gdn_fwd_args;

/* Arguments of the backward: the forward's inputs, the upstream gradients
 * dout (of o) and dST (of S_T, NULL = zero), and the gradient outputs.  The
 * backward recomputes the forward internally; no forward tape is passed.
 * dq/dk hold the sum over the value heads that share a q/k head. */
typedef struct gdn_bwd_args {
    uint32_t struct_size;
    uint32_t abi_version;
    int32_t dtype;
    int32_t B, T, Hk, Hv, dk, dv;
    int32_t num_seqs;
    uint32_t flags;
    const void* q;
    const void* k;
    const void* v;
    const float* beta;
    const float* g;
    const int32_t* cu_seqlens;
    const int32_t* cu_seqlens_host;
    const float* S0;   /* [N,Hv,dk,dv] or NULL                 */
    const void* dout;  /* [B,T,Hv,dv], dtype                   */
    const float* dST;  /* [N,Hv,dk,dv] or NULL (zero)          */
    void* dq;          /* out [B,T,Hk,dk], dtype               */
    void* dk_out;      /* out [B,T,Hk,dk], dtype               */
    void* dv_out;      /* out [B,T,Hv,dv], dtype               */
    float* dbeta;      /* out [B,T,Hv] fp32                    */
    float* dg;         /* out [B,T,Hv] fp32 (w.r.t. raw g)     */
    float* dS0;        /* out [N,Hv,dk,dv] fp32 or NULL (skip);
                          must overlap neither S0 nor dST      */
    int32_t* dev_status;
} gdn_bwd_args;

/* Bytes of device workspace gdn_chunk_fwd needs for these arguments (the
 * pointers may be NULL here; only sizes, dtype and cu_seqlens_host are read).
 * Returns GDN_OK and sets *bytes, or an argument error (a status rather than a
 * bare size, so that a bad argument cannot be mistaken for a size).  The tensor-core path
 * (bf16, dk = dv = 128) keeps three 8 KB bf16 images (T = (I + A)^-1,
 * T diag(beta Gam) and T diag(beta)) and one 8-byte gate summary per (chunk slot,
 * value head), with floor(T_total / 64) + N + 1 chunk slots; the CUDA-core path
 * keeps fp32 W, U, gamma and chunk states. */
GDN_API gdn_status gdn_chunk_fwd_workspace_size(const gdn_fwd_args* args, size_t* bytes);

/* Forward: o and (optionally) S_T from q, k, v, beta, g and (optionally) S0.
 * This is the forward kernel of the FlashQLA pages (news.hamidun.com "Qwen
 * FlashQLA ... Hopper", section "What is FlashQLA": forward pass of GDN in
 * chunked-prefill mode; its "Chunked Prefill" scenario for S0 -> S_T chaining).
 * One sequence may be split over several SMs by its gate decay (dothoosh.com
 * FlashQLA article, first innovation: gate-driven context parallelism) unless
 * GDN_FLAG_SPLIT_OFF is set.
 * workspace: device memory of at least gdn_chunk_fwd_workspace_size() bytes,
 * 256-byte aligned, caller-owned, contents irrelevant on entry.
 * stream: a cudaStream_t (CUstream) handle, or NULL for the legacy stream. */
GDN_API gdn_status gdn_chunk_fwd(const gdn_fwd_args* args, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Bytes of device workspace gdn_chunk_bwd needs: on the tensor-core path the
 * forward's images and summaries, a 32 KB bf16 entry-state image per (chunk
 * slot, value head), and with grouped heads fp32 dq / dk per value head. */
GDN_API gdn_status gdn_chunk_bwd_workspace_size(const gdn_bwd_args* args, size_t* bytes);

/* Backward: dq, dk, dv, dbeta, dg and (optionally) dS0 of the forward above
 * for upstream gradients dout and dST.  Same workspace/stream rules.  This is
 * the backward kernel of the FlashQLA pages (news.hamidun.com page, section
 * "What is FlashQLA": forward and backward passes; dothoosh.com article,
 * backward speed-up paragraph). */
GDN_API gdn_status gdn_chunk_bwd(const gdn_bwd_args* args, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Static, NUL-terminated description of a status code (never NULL).  The
 * FlashQLA pages describe no interface; this belongs to the library. */
GDN_API const char* gdn_status_string(int status);

/* Forward without a workspace argument, for callers that cannot allocate device
 * memory: code inside a framework plugin or an inference server whose device
 * memory is pooled and frozen after start-up, or any runtime that forbids
 * cudaMalloc on the request path.  (The FlashQLA pages have no counterpart; this
 * is an interface convenience of this library.)
 *
 * It computes exactly what gdn_chunk_fwd computes, always with the CUDA-core
 * kernels (as with GDN_FLAG_PORTABLE), and keeps their scratch in a
 * fixed device array of GDN_NOALLOC_SCRATCH_BYTES that is part of libgdn.so:
 * every GPU that loads the library holds it until the process exits.  It calls
 * no cudaMalloc / cudaFree.  Problems whose scratch would exceed the array are
 * rejected with GDN_ERR_TOO_LARGE before anything is enqueued (at dk = dv = 128
 * the array holds about 500 chunk x value-head pairs, e.g. 8 heads x 4000 tokens).
 *
 * All calls share the one array per device, so calls whose kernels overlap on
 * the GPU (different streams, or different threads) race on it; serialise them.
 * The kernels write every scratch byte before reading it, so nothing needs
 * clearing between calls.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current) and caches
 * it, keyed by the CUDA context; make that first call before any stream
 * capture.  After cudaDeviceReset the next call looks the address up again
 * (the new context holds a new copy of the array). */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
GDN_API gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_args* args, void* stream);

/* Arguments of one decode step: one new token for each of N sequences.
 * struct_size = sizeof(gdn_decode_args), abi_version = GDN_ABI_VERSION. */
typedef struct gdn_decode_args {
    uint32_t struct_size;
    uint32_t abi_version;
    int32_t dtype;     /* gdn_dtype of q, k, v and o                                */
    int32_t N;         /* sequences in the batch (one token each); 0 is a no-op      */
    int32_t Hk, Hv;    /* q/k heads, value heads (Hv % Hk == 0, contiguous groups)   */
    int32_t dk, dv;    /* head dims, 1..128, dv a multiple of 4                      */
    int32_t num_slots; /* states in S when state_indices != NULL (else N)            */
    uint32_t flags;    /* GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM; others ignored  */
    const void* q;     /* [N, Hk, dk] dtype                                          */
    const void* k;     /* [N, Hk, dk] dtype                                          */
    const void* v;     /* [N, Hv, dv] dtype                                          */
    const float* beta; /* [N, Hv] fp32                                               */
    const float* g;    /* [N, Hv] fp32, raw log decay, finite                        */
    float* S;          /* in/out [num_slots, Hv, dk, dv] fp32, H = S^T layout as S_T;
                          16-byte aligned                                            */
    const int32_t* state_indices; /* device int32 [N] or NULL: sequence n updates
                          slot state_indices[n] of S (a state pool, as in continuous
                          batching); a negative index skips the sequence and writes
                          zeros to its o; indices must be distinct (two sequences on
                          one slot race); NULL means slot n                          */
    void* o;           /* out [N, Hv, dv] dtype                                      */
    int32_t* dev_status; /* device int32 or NULL: GDN_ERR_DEVICE for an index
                          >= num_slots (that sequence is skipped)                    */
} gdn_decode_args;

/* Decode step: for every sequence n and value head h, with H the state in its slot,
 *     H <- exp(g) H,   H <- H + beta k (v - H^T k)^T,   o = H^T q,
 * i.e. one token of the gated delta rule applied to S in place (S_T of a prefill
 * call can be passed as S directly).  This is the token-by-token step that
 * follows chunked prefill in the inference scenarios of the FlashQLA pages
 * (news.hamidun.com "Qwen FlashQLA ... Hopper", scenario list: edge inference;
 * distributed inference with several model calls in one stream).  One kernel
 * launch; each state is read once and written once.  Asynchronous on `stream`;
 * argument errors return before anything is enqueued.  Needs no workspace. */
GDN_API gdn_status gdn_decode_step(const gdn_decode_args* args, void* stream);

/* ---- Context parallelism across GPUs (one long sequence, token shards on several
 * GPUs).  The dothoosh.com FlashQLA article (first innovation: gate-driven context
 * parallelism; its million-token paragraph) splits one long sequence automatically
 * among processing units; across GPUs a shard needs the state its sequence carries
 * into it.  Two ways to get it, both per (sequence, value head):
 *  - the gate-driven way: start the shard a few chunks early (a halo of the previous
 *    shard's last tokens) from a zero state; valid when the halo's summed log decay
 *    is at most log(eps) and every halo token keeps 0 <= beta |k|^2 <= 2 (each
 *    token's state map then has norm <= exp(g_t)), gdn_halo_check below;
 *  - the exact way: every shard's tokens map its entry state affinely,
 *    H_exit = M H_entry + B (M = the product of the tokens' maps, dk x dk; B = the
 *    exit state from a zero entry), and the entry state of shard r is the fold of
 *    shards 0..r-1 applied to S0, X <- M_j X + B_j in order: gdn_affine_combine below.
 * The shards' folds (M from a forward with v = 0 and S0 = [I | 0], B from a forward
 * with S0 = 0) and the collectives belong to the caller (the Python package's
 * cp_chunk_fwd). */

/* One step of the affine fold, per (sequence n, value head h):
 *     X <- M X + B      (M [dk][dk], X and B [dk][dv], fp32, row-major).
 * struct_size = sizeof(gdn_combine_args), abi_version = GDN_ABI_VERSION. */
typedef struct gdn_combine_args {
    uint32_t struct_size;
    uint32_t abi_version;
    int32_t N, Hv;    /* sequences and value heads (N * Hv states); 0 is a no-op      */
    int32_t dk, dv;   /* 1..128                                                      */
    const float* M;   /* [N, Hv, dk, dk]                                             */
    const float* B;   /* [N, Hv, dk, dv] or NULL (zero)                              */
    float* X;         /* in / out [N, Hv, dk, dv]; must overlap neither M nor B
                         (GDN_ERR_INVALID_ARG); X, M and B 16-byte aligned            */
} gdn_combine_args;
/* One launch; asynchronous on `stream`; argument errors return before anything is
 * enqueued.  fp32 arithmetic (fused multiply-adds in row order j = 0..dk-1). */
GDN_API gdn_status gdn_affine_combine(const gdn_combine_args* args, void* stream);

/* Whether a halo of tokens can stand in for everything before it, per value head:
 * ok[h] = 1 when sum_t g[t][h] <= log_eps and 0 <= beta[t][h] |k[t][h / G]|^2 <= 2 for
 * every halo token t (G = Hv / Hk; with GDN_FLAG_GATE_LOGITS g and beta are mapped
 * first, with GDN_FLAG_QK_L2NORM k is normalised first, as in the forward), else 0.
 * The gate-driven split of a sequence (dothoosh.com FlashQLA article, first
 * innovation) takes this test for its warm-up across SMs; across GPUs the halo is
 * the previous shard's last tokens.  struct_size = sizeof(gdn_halo_args). */
typedef struct gdn_halo_args {
    uint32_t struct_size;
    uint32_t abi_version;
    int32_t dtype;       /* gdn_dtype of k                                             */
    int32_t T;           /* halo tokens (0: every head fails, no halo to stand in)     */
    int32_t Hk, Hv, dk;  /* heads as in the forward, dk 1..128                         */
    uint32_t flags;      /* GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM; others ignored  */
    float log_eps;       /* bound on the summed log decay (the forward uses -30 ln 2) */
    const void* k;       /* [T, Hk, dk] dtype                                          */
    const float* beta;   /* [T, Hv]                                                    */
    const float* g;      /* [T, Hv]                                                    */
    int32_t* ok;         /* out [Hv]                                                   */
    float* log_decay;    /* out [Hv] (the summed log decay) or NULL                    */
} gdn_halo_args;
/* One launch; asynchronous on `stream`; argument errors return before anything is
 * enqueued. */
GDN_API gdn_status gdn_halo_check(const gdn_halo_args* args, void* stream);

/* Number of kernel launches gdn_chunk_fwd / gdn_chunk_bwd enqueue for these
 * arguments (a pure function of the arguments; -1 on an argument error).  The
 * FlashQLA pages describe no interface; this is for launch accounting. */
GDN_API int gdn_chunk_fwd_launch_count(const gdn_fwd_args* args);
GDN_API int gdn_chunk_bwd_launch_count(const gdn_bwd_args* args);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
