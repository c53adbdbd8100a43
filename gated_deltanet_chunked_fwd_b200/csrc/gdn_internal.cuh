// gdn_internal.cuh -- types shared by the entry points and the kernels of libgdn.
//
// Notation (one sequence, one value head, one chunk of n <= C = 64 tokens):
//   gamma = in-chunk inclusive cumsum of g,  Gam = exp(gamma),
//   E[r][s] = exp(gamma_r - gamma_s),        H = S^T  (dk x dv state at chunk entry)
//   A = strictly-lower(diag(beta) (K K^T o E)),  T = (I + A)^-1        (WY / UT transform)
//   W = T diag(beta Gam) K,  Ut = T diag(beta) V,  U = Ut - W H          (corrected values)
//   O = diag(Gam) Q H + lower-incl(Q K^T o E) U                           (chunk output)
//   H' = Gam_n H + Kd^T U,  Kd = diag(exp(gamma_n - gamma)) K            (state passing)
// This is the gated delta rule S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// o_t = S_t q_t (the GDN layer of the FlashQLA pages, news.hamidun.com "What is FlashQLA"),
// regrouped into chunks; the chunk-level equations are derived from the rule and
// checked against the token-by-token float64 oracle.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

constexpr int kChunk = GDN_CHUNK;  // 64
constexpr int kMaxHead = 128;       // largest dk / dv

// One call's problem description, in device-usable form (passed by value).
struct Problem {
    int dtype;          // GDN_F32 / GDN_BF16
    int N;              // sequences
    int T;              // tokens per sequence (fixed length) or total tokens (varlen)
    int64_t T_total;    // total tokens (= B*T or cu[N])
    int Hk, Hv, dk, dv, group;  // group = Hv / Hk
    const void* q;
    const void* k;
    const void* v;
    const float* beta;
    const float* g;
    const int32_t* cu;  // device offsets or nullptr (fixed length)
    const float* S0;
    void* o;
    float* ST;
    int32_t* status;
    int64_t num_chunks;  // sum over sequences of ceil(len / 64)
    int gate_logits;     // GDN_FLAG_GATE_LOGITS: beta and g hold logits / pre-activations
    int qk_norm;         // GDN_FLAG_QK_L2NORM: q and k rows are normalised before use
};

constexpr float kL2Eps = 1e-6f;  // GDN_FLAG_QK_L2NORM: x / max(|x|_2, kL2Eps)

// GDN_FLAG_QK_L2NORM on rows held in shared memory as fp32: X[r][0, dk) <- X[r] / max(|X[r]|_2,
// kL2Eps) for r < rows, one warp per row; the caller synchronises before and after.
__device__ __forceinline__ void l2norm_rows_smem(float* X, int rows, int dk) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int r = warp; r < rows; r += nw) {
        float ss = 0.f;
        for (int i = lane; i < dk; i += 32) ss += X[r * dk + i] * X[r * dk + i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = 1.f / fmaxf(sqrtf(ss), kL2Eps);
        for (int i = lane; i < dk; i += 32) X[r * dk + i] *= inv;
    }
}

// Raw gates (GDN_FLAG_GATE_LOGITS): beta = sigmoid(b) and g = -softplus(a) = -log(1 + e^a), the
// latter as -(max(a, 0) + log1p(e^-|a|)), which neither overflows nor loses small values; the
// identity maps otherwise.  Padding tokens keep their plain zeros (callers apply the maps to
// loaded values only).
__device__ __forceinline__ float gate_beta(float b, int logits) { return logits ? 1.f / (1.f + expf(-b)) : b; }
__device__ __forceinline__ float gate_g(float a, int logits) {
    return logits ? -(fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)))) : a;
}
// Chain rule back to the raw gates: d/db sigmoid(b) = beta (1 - beta) (from the mapped beta),
// d/da -softplus(a) = -sigmoid(a).
__device__ __forceinline__ float gate_beta_grad(float dbeta, float beta, int logits) {
    return logits ? dbeta * beta * (1.f - beta) : dbeta;
}
__device__ __forceinline__ float gate_g_grad(float dg, float a, int logits) {
    return logits ? -dg / (1.f + expf(-a)) : dg;
}

// Per-chunk lookup built on the device from cu_seqlens (or arithmetic).
struct ChunkTable {
    int32_t* seq;        // [num_chunks] sequence of the chunk
    int32_t* t0;         // [num_chunks] first token (packed index)
    int32_t* len;        // [num_chunks] tokens in the chunk, 1..64
    int32_t* seq_chunk0; // [N + 1] first chunk of each sequence
};

// Backward extras.
struct BwdProblem {
    Problem f;
    const void* dout;
    const float* dST;
    void* dq;
    void* dk;
    void* dv;
    float* dbeta;
    float* dg;
    float* dS0;
};

// Device status helper: first error wins.
__device__ __forceinline__ void report(int32_t* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---- host-side planning --------------------------------------------------
struct FwdPlan {
    Problem p;
    bool use_tc;         // tensor-core fused kernel
    const int32_t* cu_host;  // host copy of cu_seqlens (or nullptr)
    int split_mode;      // 0 auto, 1 off, 2 force
    // workspace carve-up (byte offsets); sizes are 0 when unused
    size_t off_table, off_W, off_U, off_gam, off_Hc, total;
    int launches;
};

gdn_status plan_fwd(const gdn_fwd_args* a, FwdPlan* plan);
gdn_status launch_fwd_simt(const FwdPlan& plan, char* ws, cudaStream_t s);
gdn_status launch_fwd_tc(const FwdPlan& plan, char* ws, cudaStream_t s);
size_t tc_fwd_workspace(const Problem& p, const int32_t* cu_host, int split_mode);
size_t wy_tc_workspace(const Problem& p);
size_t wy_tc_summary_offset(const Problem& p);
// WY + fused kernel in replay mode: bf16 H^T entry-state image (32 KB) of every chunk, by
// (image slot, value head), into himg; `ws` holds the WY outputs (wy_tc_workspace bytes);
// split_mode as in FwdPlan; the WY launch also zeroes the nrflags int32 flags at rflags (the
// backward's adjoint scan)
gdn_status launch_replay_tc(const Problem& p, const int32_t* cu_host, int split_mode, char* ws,
                            uint8_t* himg, cudaStream_t s, int32_t* rflags, int nrflags);
int tc_fwd_launches(const Problem& p);
bool tc_fwd_supported(const Problem& p);

struct BwdPlan {
    BwdProblem b;
    bool use_tc;  // tensor-core backward
    const int32_t* cu_host;  // host copy of cu_seqlens (or nullptr)
    int split_mode;          // 0 auto, 1 off, 2 force
    size_t off_table, off_W, off_U, off_gam, off_Hc, off_dHc, off_dU, off_dqw, off_dkw, total;
    int launches;
};
gdn_status plan_bwd(const gdn_bwd_args* a, BwdPlan* plan);
gdn_status launch_bwd_simt(const BwdPlan& plan, char* ws, cudaStream_t s);
gdn_status launch_bwd_reduce(const BwdProblem& b, const float* dqw, const float* dkw, cudaStream_t s);
bool tc_bwd_supported(const Problem& p);
size_t tc_bwd_workspace(const Problem& p, const int32_t* cu_host, int split_mode, size_t* off_himg,
                        size_t* off_timg, size_t* off_dqw, size_t* off_dkw);
int tc_bwd_launches(const Problem& p, const int32_t* cu_host, int split_mode);
gdn_status launch_bwd_tc(const BwdPlan& plan, char* ws, cudaStream_t s);

// shared SIMT pieces (also used by the backward's forward recompute)
gdn_status launch_chunk_table(const Problem& p, const ChunkTable& ct, cudaStream_t s);
gdn_status launch_simt_wy(const Problem& p, const ChunkTable& ct, float* W, float* U, float* gam,
                          cudaStream_t s);
gdn_status launch_simt_state(const Problem& p, const ChunkTable& ct, const float* W, float* U,
                             const float* gam, float* Hc, float* ST, cudaStream_t s);
gdn_status launch_simt_output(const Problem& p, const ChunkTable& ct, const float* U,
                              const float* gam, const float* Hc, cudaStream_t s);

// decode step (gdn_decode.cu)
gdn_status plan_decode(const gdn_decode_args* a);
gdn_status launch_decode(const gdn_decode_args* a, cudaStream_t s);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace gdn
