// gdn_simt_fwd.cu -- CUDA-core (SIMT) forward of the chunked gated delta rule.
//
// The portable path: fp32 arithmetic on CUDA cores for every supported shape
// (dk, dv <= 128, fp32 or bf16 tensors).  It is the path for fp32 inputs, and
// the three-kernel split it uses mirrors the three subsystems of the chunked
// forward:
//   simt_wy_kernel     per (chunk, head), parallel: gamma, A, T = (I + A)^-1,
//                      W = T diag(beta Gam) K, Ut = T diag(beta) V
//   simt_state_kernel  per (sequence, head, 32 state columns), sequential over
//                      chunks: H_c (chunk-entry state), U = Ut - W H_c,
//                      H <- Gam_n H + Kd^T U; final state S_T
//   simt_output_kernel per (chunk, head), parallel: O = diag(Gam) Q H_c + P U
// Columns of the state never interact (the delta rule mixes the state only
// along dk), so the sequential state scan splits over dv with no exchange.
#include "gdn_dtype.cuh"
#include "gdn_internal.cuh"

namespace gdn {

// Sequence bounds [bos, eos) from cu_seqlens or the fixed length.
__device__ __forceinline__ void seq_bounds(const Problem& p, int n, int64_t& bos, int64_t& eos) {
    if (p.cu) {
        bos = p.cu[n];
        eos = p.cu[n + 1];
        if (eos < bos) eos = bos;
    } else {
        bos = (int64_t)n * p.T;
        eos = bos + p.T;
    }
}

// One block builds the chunk table: chunk counts per sequence, a block-wide
// exclusive scan, then each thread writes the entries of its sequences.
__global__ void __launch_bounds__(1024) chunk_table_kernel(Problem p, ChunkTable ct) {
    __shared__ int64_t part[1024];
    const int nt = blockDim.x, tid = threadIdx.x;
    const int per = (p.N + nt - 1) / nt;
    const int a = min(p.N, tid * per), b = min(p.N, a + per);
    int64_t local = 0;
    for (int n = a; n < b; ++n) {
        int64_t bos, eos;
        seq_bounds(p, n, bos, eos);
        local += (eos - bos + kChunk - 1) / kChunk;
    }
    part[tid] = local;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {  // inclusive Hillis-Steele scan
        int64_t add = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += add;
        __syncthreads();
    }
    int64_t base = part[tid] - local;
    for (int n = a; n < b; ++n) {
        int64_t bos, eos;
        seq_bounds(p, n, bos, eos);
        ct.seq_chunk0[n] = (int32_t)min(base, p.num_chunks);
        for (int64_t t = bos; t < eos; t += kChunk, ++base) {
            if (base >= p.num_chunks) {  // device offsets disagree with the host copy
                report(p.status, GDN_ERR_DEVICE);
                break;
            }
            ct.seq[base] = n;
            ct.t0[base] = (int32_t)t;
            ct.len[base] = (int32_t)(eos - t < kChunk ? eos - t : kChunk);
        }
    }
    if (tid == nt - 1) {
        ct.seq_chunk0[p.N] = (int32_t)min(part[nt - 1], p.num_chunks);
        if (part[nt - 1] != p.num_chunks) report(p.status, GDN_ERR_DEVICE);
    }
}

// ---------------------------------------------------------------- WY / UT
template <typename Tin>
__global__ void __launch_bounds__(256) simt_wy_kernel(Problem p, ChunkTable ct, float* W, float* U,
                                                      float* gam) {
    const int c = blockIdx.x, h = blockIdx.y, hk = h / p.group;
    const int dk = p.dk, dv = p.dv;
    const int t0 = ct.t0[c], n = ct.len[c];
    extern __shared__ float sm[];
    float* Ks = sm;                 // [64][dk]
    float* A = Ks + kChunk * dk;    // [64][64]
    float* Tm = A + kChunk * kChunk;  // [64][64]
    float* bs = Tm + kChunk * kChunk;  // beta
    float* gs = bs + kChunk;        // gamma
    float* bgs = gs + kChunk;       // beta * Gam
    const Tin* kp = (const Tin*)p.k;
    const Tin* vp = (const Tin*)p.v;
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        Ks[idx] = r < n ? to_f(kp[((int64_t)(t0 + r) * p.Hk + hk) * dk + i]) : 0.f;
    }
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        bs[r] = r < n ? gate_beta(p.beta[(int64_t)(t0 + r) * p.Hv + h], p.gate_logits) : 0.f;
        gs[r] = r < n ? gate_g(p.g[(int64_t)(t0 + r) * p.Hv + h], p.gate_logits) : 0.f;  // padding: g = 0
    }
    __syncthreads();
    if (p.qk_norm) {  // raw k rows: normalised before use
        l2norm_rows_smem(Ks, kChunk, dk);
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        float acc = 0.f;
        for (int r = 0; r < kChunk; ++r) {
            acc += gs[r];
            gs[r] = acc;
        }
    }
    __syncthreads();
    if (threadIdx.x < kChunk) bgs[threadIdx.x] = bs[threadIdx.x] * expf(gs[threadIdx.x]);
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float a = 0.f;
        if (s < r && r < n) {
            float d = 0.f;
            for (int i = 0; i < dk; ++i) d += Ks[r * dk + i] * Ks[s * dk + i];
            a = bs[r] * d * expf(gs[r] - gs[s]);
        }
        A[idx] = a;
    }
    __syncthreads();
    // T = (I + A)^-1 by forward substitution, one column per thread.
    if (threadIdx.x < kChunk) {
        const int col = threadIdx.x;
        for (int r = 0; r < kChunk; ++r) {
            float val;
            if (r < col) {
                val = 0.f;
            } else if (r == col) {
                val = 1.f;
            } else {
                float s = 0.f;
                for (int j = col; j < r; ++j) s += A[r * kChunk + j] * Tm[j * kChunk + col];
                val = -s;
            }
            Tm[r * kChunk + col] = val;
        }
    }
    __syncthreads();
    const int64_t ch = (int64_t)c * p.Hv + h;
    float* Wc = W + ch * kChunk * dk;
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        float acc = 0.f;
        for (int s = 0; s <= r; ++s) acc += Tm[r * kChunk + s] * bgs[s] * Ks[s * dk + i];
        Wc[idx] = acc;
    }
    float* Uc = U + ch * kChunk * dv;
    for (int idx = threadIdx.x; idx < kChunk * dv; idx += blockDim.x) {
        const int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        const int smax = min(r, n - 1);
        for (int s = 0; s <= smax; ++s)
            acc += Tm[r * kChunk + s] * bs[s] * to_f(vp[((int64_t)(t0 + s) * p.Hv + h) * dv + j]);
        Uc[idx] = acc;
    }
    if (threadIdx.x < kChunk) gam[ch * kChunk + threadIdx.x] = gs[threadIdx.x];
}

// ------------------------------------------------------------ state scan
constexpr int kSlice = 32;  // state columns per block

template <typename Tin>
__global__ void __launch_bounds__(256) simt_state_kernel(Problem p, ChunkTable ct, const float* W,
                                                         float* U, const float* gam, float* Hc,
                                                         float* ST) {
    const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSlice, hk = h / p.group;
    const int dk = p.dk, dv = p.dv, sw = min(kSlice, dv - j0);
    extern __shared__ float sm[];
    float* Hs = sm;                  // [dk][32]
    float* Us = Hs + dk * kSlice;    // [64][32]
    float* Kd = Us + kChunk * kSlice;  // [64][dk]
    float* gs = Kd + kChunk * dk;    // [64]
    const Tin* kp = (const Tin*)p.k;
    const int64_t sbase = ((int64_t)n * p.Hv + h) * dk * dv;
    for (int idx = threadIdx.x; idx < dk * kSlice; idx += blockDim.x) {
        const int i = idx / kSlice, jj = idx % kSlice;
        Hs[idx] = (jj < sw && p.S0) ? p.S0[sbase + (int64_t)i * dv + j0 + jj] : 0.f;
    }
    const int c_begin = ct.seq_chunk0[n], c_end = ct.seq_chunk0[n + 1];
    for (int c = c_begin; c < c_end; ++c) {
        const int t0 = ct.t0[c], len = ct.len[c];
        const int64_t ch = (int64_t)c * p.Hv + h;
        if (threadIdx.x < kChunk) gs[threadIdx.x] = gam[ch * kChunk + threadIdx.x];
        __syncthreads();
        const float gl = gs[kChunk - 1];
        if (!p.qk_norm) {
            for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
                const int r = idx / dk, i = idx % dk;
                Kd[idx] = r < len ? to_f(kp[((int64_t)(t0 + r) * p.Hk + hk) * dk + i]) * expf(gl - gs[r])
                                  : 0.f;
            }
        } else {  // raw k rows: normalised, then scaled by the decay
            for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
                const int r = idx / dk, i = idx % dk;
                Kd[idx] = r < len ? to_f(kp[((int64_t)(t0 + r) * p.Hk + hk) * dk + i]) : 0.f;
            }
            __syncthreads();
            l2norm_rows_smem(Kd, kChunk, dk);
            __syncthreads();
            for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
                const int r = idx / dk;
                Kd[idx] *= r < len ? expf(gl - gs[r]) : 0.f;
            }
        }
        float* Hcc = Hc + ch * dk * dv;
        for (int idx = threadIdx.x; idx < dk * kSlice; idx += blockDim.x) {
            const int i = idx / kSlice, jj = idx % kSlice;
            if (jj < sw) Hcc[(int64_t)i * dv + j0 + jj] = Hs[idx];
        }
        // U = Ut - W H
        const float* Wc = W + ch * kChunk * dk;
        float* Uc = U + ch * kChunk * dv;
        for (int idx = threadIdx.x; idx < kChunk * kSlice; idx += blockDim.x) {
            const int r = idx / kSlice, jj = idx % kSlice;
            float acc = 0.f;
            if (jj < sw) {
                acc = Uc[r * dv + j0 + jj];
                for (int i = 0; i < dk; ++i) acc -= Wc[r * dk + i] * Hs[i * kSlice + jj];
                Uc[r * dv + j0 + jj] = acc;
            }
            Us[idx] = acc;
        }
        __syncthreads();
        // H <- Gam_n H + Kd^T U
        const float Gn = expf(gl);
        for (int idx = threadIdx.x; idx < dk * kSlice; idx += blockDim.x) {
            const int i = idx / kSlice, jj = idx % kSlice;
            float acc = Gn * Hs[idx];
            for (int r = 0; r < kChunk; ++r) acc += Kd[r * dk + i] * Us[r * kSlice + jj];
            Hs[idx] = acc;
        }
        __syncthreads();
    }
    if (ST) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < dk * kSlice; idx += blockDim.x) {
            const int i = idx / kSlice, jj = idx % kSlice;
            if (jj < sw) ST[sbase + (int64_t)i * dv + j0 + jj] = Hs[idx];
        }
    }
}

// ---------------------------------------------------------------- output
template <typename Tin>
__global__ void __launch_bounds__(256) simt_output_kernel(Problem p, ChunkTable ct, const float* U,
                                                          const float* gam, const float* Hc) {
    const int c = blockIdx.x, h = blockIdx.y, hk = h / p.group;
    const int dk = p.dk, dv = p.dv;
    const int t0 = ct.t0[c], n = ct.len[c];
    extern __shared__ float sm[];
    float* Qs = sm;                   // [64][dk]
    float* Ks = Qs + kChunk * dk;     // [64][dk]
    float* P = Ks + kChunk * dk;      // [64][64]
    float* gs = P + kChunk * kChunk;  // [64]
    const Tin* qp = (const Tin*)p.q;
    const Tin* kp = (const Tin*)p.k;
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        const int64_t off = ((int64_t)(t0 + r) * p.Hk + hk) * dk + i;
        Qs[idx] = r < n ? to_f(qp[off]) : 0.f;
        Ks[idx] = r < n ? to_f(kp[off]) : 0.f;
    }
    const int64_t ch = (int64_t)c * p.Hv + h;
    if (threadIdx.x < kChunk) gs[threadIdx.x] = gam[ch * kChunk + threadIdx.x];
    __syncthreads();
    if (p.qk_norm) {  // raw q and k rows: normalised before use
        l2norm_rows_smem(Qs, kChunk, dk);
        l2norm_rows_smem(Ks, kChunk, dk);
        __syncthreads();
    }
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float v = 0.f;
        if (s <= r && r < n) {
            float d = 0.f;
            for (int i = 0; i < dk; ++i) d += Qs[r * dk + i] * Ks[s * dk + i];
            v = d * expf(gs[r] - gs[s]);
        }
        P[idx] = v;
    }
    __syncthreads();
    const float* Hcc = Hc + ch * dk * dv;
    const float* Uc = U + ch * kChunk * dv;
    Tin* op = (Tin*)p.o;
    for (int idx = threadIdx.x; idx < kChunk * dv; idx += blockDim.x) {
        const int r = idx / dv, j = idx % dv;
        if (r >= n) continue;
        float qh = 0.f;
        for (int i = 0; i < dk; ++i) qh += Qs[r * dk + i] * Hcc[(int64_t)i * dv + j];
        float pu = 0.f;
        for (int s = 0; s <= r; ++s) pu += P[r * kChunk + s] * Uc[s * dv + j];
        store_as(op + ((int64_t)(t0 + r) * p.Hv + h) * dv + j, expf(gs[r]) * qh + pu);
    }
}

// ------------------------------------------------------------- launchers
static gdn_status check_launch() {
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename K>
static gdn_status set_smem(K kernel, size_t bytes) {
    if (bytes > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
            cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

gdn_status launch_chunk_table(const Problem& p, const ChunkTable& ct, cudaStream_t s) {
    chunk_table_kernel<<<1, 1024, 0, s>>>(p, ct);
    return check_launch();
}

gdn_status launch_simt_wy(const Problem& p, const ChunkTable& ct, float* W, float* U, float* gam,
                          cudaStream_t s) {
    const size_t smem = sizeof(float) * (kChunk * p.dk + 2 * kChunk * kChunk + 3 * kChunk);
    dim3 grid((unsigned)p.num_chunks, p.Hv);
    if (p.dtype == GDN_BF16) {
        if (set_smem(simt_wy_kernel<__nv_bfloat16>, smem)) return GDN_ERR_CUDA;
        simt_wy_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(p, ct, W, U, gam);
    } else {
        if (set_smem(simt_wy_kernel<float>, smem)) return GDN_ERR_CUDA;
        simt_wy_kernel<float><<<grid, 256, smem, s>>>(p, ct, W, U, gam);
    }
    return check_launch();
}

gdn_status launch_simt_state(const Problem& p, const ChunkTable& ct, const float* W, float* U,
                             const float* gam, float* Hc, float* ST, cudaStream_t s) {
    const size_t smem =
        sizeof(float) * (p.dk * kSlice + kChunk * kSlice + kChunk * p.dk + kChunk);
    dim3 grid(p.N, p.Hv, (p.dv + kSlice - 1) / kSlice);
    if (p.dtype == GDN_BF16) {
        if (set_smem(simt_state_kernel<__nv_bfloat16>, smem)) return GDN_ERR_CUDA;
        simt_state_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(p, ct, W, U, gam, Hc, ST);
    } else {
        if (set_smem(simt_state_kernel<float>, smem)) return GDN_ERR_CUDA;
        simt_state_kernel<float><<<grid, 256, smem, s>>>(p, ct, W, U, gam, Hc, ST);
    }
    return check_launch();
}

gdn_status launch_simt_output(const Problem& p, const ChunkTable& ct, const float* U,
                              const float* gam, const float* Hc, cudaStream_t s) {
    const size_t smem = sizeof(float) * (2 * kChunk * p.dk + kChunk * kChunk + kChunk);
    dim3 grid((unsigned)p.num_chunks, p.Hv);
    if (p.dtype == GDN_BF16) {
        if (set_smem(simt_output_kernel<__nv_bfloat16>, smem)) return GDN_ERR_CUDA;
        simt_output_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(p, ct, U, gam, Hc);
    } else {
        if (set_smem(simt_output_kernel<float>, smem)) return GDN_ERR_CUDA;
        simt_output_kernel<float><<<grid, 256, smem, s>>>(p, ct, U, gam, Hc);
    }
    return check_launch();
}

// Workspace carve-up shared with the planner: table | W | U | gamma | Hc.
gdn_status launch_fwd_simt(const FwdPlan& plan, char* ws, cudaStream_t s) {
    const Problem& p = plan.p;
    const int64_t nc = p.num_chunks;
    ChunkTable ct;
    ct.seq = (int32_t*)(ws + plan.off_table);
    ct.t0 = ct.seq + nc;
    ct.len = ct.t0 + nc;
    ct.seq_chunk0 = ct.len + nc;
    float* W = (float*)(ws + plan.off_W);
    float* U = (float*)(ws + plan.off_U);
    float* gam = (float*)(ws + plan.off_gam);
    float* Hc = (float*)(ws + plan.off_Hc);
    gdn_status st = launch_chunk_table(p, ct, s);
    if (st) return st;
    if (nc > 0) {
        if ((st = launch_simt_wy(p, ct, W, U, gam, s))) return st;
    }
    if ((st = launch_simt_state(p, ct, W, U, gam, Hc, p.ST, s))) return st;
    if (nc > 0) {
        if ((st = launch_simt_output(p, ct, U, gam, Hc, s))) return st;
    }
    return GDN_OK;
}

}  // namespace gdn
