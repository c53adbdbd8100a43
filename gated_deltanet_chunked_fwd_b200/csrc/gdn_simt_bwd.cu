// gdn_simt_bwd.cu -- CUDA-core (SIMT) backward of the chunked gated delta rule.
//
// The backward (FlashQLA pages: dothoosh.com article, opening paragraph, backward
// pass; news.hamidun.com page, "large-scale pretraining" scenario) is the
// reverse-mode adjoint of the chunk equations listed in gdn_internal.cuh:
//   1. forward recompute (shared kernels): gamma, W, Ut, then the state scan
//      writes every chunk-entry state H_c and the corrected values U;
//   2. simt_bwd_dstate_kernel, per (sequence, head, 32 state columns),
//      sequential over chunks in reverse: with dH the adjoint of the chunk's
//      exit state,  dU = P^T dO + Kd dH  and
//      dH <- Gam_n dH + (diag(Gam) Q)^T dO - W^T dU;  dS0 is the final dH;
//   3. simt_bwd_chunk_kernel, per (chunk, value head), parallel: every
//      per-token gradient of the chunk from (H_c, dH_c, U, dU);
//   4. simt_bwd_reduce_kernel: sums dq / dk over the value heads of a group.
// Per chunk (see the chunk kernel for the order of evaluation):
//   dQs = diag(Gam) dO H^T       dP  = lower-incl(dO U^T)
//   dW  = -dU H^T                dT  = dW Kb^T + dU Vb^T   (Kb = diag(beta Gam) K, Vb = diag(beta) V)
//   dA  = strictly-lower(-T^T dT T^T),   G = dA o E o beta_row
//   dq  = dQs + (dP o E) K
//   dk  = (dP o E)^T Q + diag(exp(gamma_n - gamma)) U dH^T + diag(beta Gam) T^T dW + (G + G^T) K
//   dv  = diag(beta) T^T dU
//   dbeta_r = sum_s (dA o K K^T o E)_rs + Gam_r (T^T dW)_r . k_r + (T^T dU)_r . v_r
//   dgamma  = rowdot(Q, dQs) + rowsum - colsum (dP o P) + rowsum - colsum (dA o A)
//             + rowdot(T^T dW, Kb) - rowdot(Kd, U dH^T)
//             + [sum(Kd o U dH^T) + Gam_n <dH, H>] at the last token
//   dg = reverse in-chunk cumsum of dgamma.
#include <algorithm>

#include "gdn_dtype.cuh"
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kSliceB = 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ------------------------------------------------------- reverse state scan
template <typename Tin>
__global__ void __launch_bounds__(256) simt_bwd_dstate_kernel(BwdProblem b, ChunkTable ct,
                                                              const float* W, const float* gam,
                                                              float* dHc, float* dU) {
    const Problem& p = b.f;
    const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSliceB, hk = h / p.group;
    const int dk = p.dk, dv = p.dv, sw = min(kSliceB, dv - j0);
    extern __shared__ float sm[];
    float* Qs = sm;                     // [64][dk]
    float* Ks = Qs + kChunk * dk;       // [64][dk]
    float* P = Ks + kChunk * dk;        // [64][64]
    float* dHs = P + kChunk * kChunk;   // [dk][32]
    float* dUs = dHs + dk * kSliceB;    // [64][32]
    float* dOs = dUs + kChunk * kSliceB;  // [64][32]
    float* gs = dOs + kChunk * kSliceB;  // [64]
    const Tin* qp = (const Tin*)p.q;
    const Tin* kp = (const Tin*)p.k;
    const Tin* dop = (const Tin*)b.dout;
    const int64_t sbase = ((int64_t)n * p.Hv + h) * dk * dv;
    for (int idx = threadIdx.x; idx < dk * kSliceB; idx += blockDim.x) {
        const int i = idx / kSliceB, jj = idx % kSliceB;
        dHs[idx] = (jj < sw && b.dST) ? b.dST[sbase + (int64_t)i * dv + j0 + jj] : 0.f;
    }
    const int c_begin = ct.seq_chunk0[n], c_end = ct.seq_chunk0[n + 1];
    for (int c = c_end - 1; c >= c_begin; --c) {
        const int t0 = ct.t0[c], len = ct.len[c];
        const int64_t ch = (int64_t)c * p.Hv + h;
        if (threadIdx.x < kChunk) gs[threadIdx.x] = gam[ch * kChunk + threadIdx.x];
        for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
            const int r = idx / dk, i = idx % dk;
            const int64_t off = ((int64_t)(t0 + r) * p.Hk + hk) * dk + i;
            Qs[idx] = r < len ? to_f(qp[off]) : 0.f;
            Ks[idx] = r < len ? to_f(kp[off]) : 0.f;
        }
        if (p.qk_norm) {  // raw q and k rows: normalised before use
            __syncthreads();
            l2norm_rows_smem(Qs, kChunk, dk);
            l2norm_rows_smem(Ks, kChunk, dk);
        }
        for (int idx = threadIdx.x; idx < kChunk * kSliceB; idx += blockDim.x) {
            const int r = idx / kSliceB, jj = idx % kSliceB;
            dOs[idx] = (r < len && jj < sw) ? to_f(dop[((int64_t)(t0 + r) * p.Hv + h) * dv + j0 + jj])
                                            : 0.f;
        }
        float* dHcc = dHc + ch * dk * dv;
        for (int idx = threadIdx.x; idx < dk * kSliceB; idx += blockDim.x) {
            const int i = idx / kSliceB, jj = idx % kSliceB;
            if (jj < sw) dHcc[(int64_t)i * dv + j0 + jj] = dHs[idx];
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
            const int r = idx / kChunk, s = idx % kChunk;
            float v = 0.f;
            if (s <= r && r < len) {
                float d = 0.f;
                for (int i = 0; i < dk; ++i) d += Qs[r * dk + i] * Ks[s * dk + i];
                v = d * expf(gs[r] - gs[s]);
            }
            P[idx] = v;
        }
        __syncthreads();
        const float gl = gs[kChunk - 1];
        // dU = P^T dO + Kd dH
        float* dUc = dU + ch * kChunk * dv;
        for (int idx = threadIdx.x; idx < kChunk * kSliceB; idx += blockDim.x) {
            const int r = idx / kSliceB, jj = idx % kSliceB;
            float acc = 0.f;
            if (r < len && jj < sw) {
                for (int s = r; s < len; ++s) acc += P[s * kChunk + r] * dOs[s * kSliceB + jj];
                float kd = 0.f;
                for (int i = 0; i < dk; ++i) kd += Ks[r * dk + i] * dHs[i * kSliceB + jj];
                acc += expf(gl - gs[r]) * kd;
                dUc[r * dv + j0 + jj] = acc;
            } else if (jj < sw) {
                dUc[r * dv + j0 + jj] = 0.f;
            }
            dUs[idx] = acc;
        }
        __syncthreads();
        // dH <- Gam_n dH + (diag(Gam) Q)^T dO - W^T dU
        const float* Wc = W + ch * kChunk * dk;
        const float Gn = expf(gl);
        for (int idx = threadIdx.x; idx < dk * kSliceB; idx += blockDim.x) {
            const int i = idx / kSliceB, jj = idx % kSliceB;
            float acc = Gn * dHs[idx];
            for (int r = 0; r < len; ++r)
                acc += expf(gs[r]) * Qs[r * dk + i] * dOs[r * kSliceB + jj] -
                       Wc[r * dk + i] * dUs[r * kSliceB + jj];
            dHs[idx] = acc;
        }
        __syncthreads();
    }
    if (b.dS0) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < dk * kSliceB; idx += blockDim.x) {
            const int i = idx / kSliceB, jj = idx % kSliceB;
            if (jj < sw) b.dS0[sbase + (int64_t)i * dv + j0 + jj] = dHs[idx];
        }
    }
}

// ------------------------------------------------------ per-chunk gradients
template <typename Tin>
__global__ void __launch_bounds__(256) simt_bwd_chunk_kernel(BwdProblem b, ChunkTable ct,
                                                             const float* U, const float* gam,
                                                             const float* Hc, const float* dHc,
                                                             const float* dU, float* dqw,
                                                             float* dkw) {
    const Problem& p = b.f;
    const int c = blockIdx.x, h = blockIdx.y, hk = h / p.group;
    const int dk = p.dk, dv = p.dv;
    const int t0 = ct.t0[c], n = ct.len[c];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
    extern __shared__ float sm[];
    float* Qs = sm;                       // [64][dk]
    float* Ks = Qs + kChunk * dk;         // [64][dk]
    float* Wb = Ks + kChunk * dk;         // [64][dk]  dW
    float* TW = Wb + kChunk * dk;         // [64][dk]  T^T dW
    float* KE = TW + kChunk * dk;         // [64][64]  (K K^T o E), strictly lower
    float* Tm = KE + kChunk * kChunk;     // [64][64]  T
    float* Pb = Tm + kChunk * kChunk;     // [64][64]  P, later Y = dT T^T
    float* dP = Pb + kChunk * kChunk;     // [64][64]  dP, later dP o E
    float* dA = dP + kChunk * kChunk;     // [64][64]  dT, later dA, later G
    float* bs = dA + kChunk * kChunk;     // beta
    float* gs = bs + kChunk;              // gamma
    float* Gs = gs + kChunk;              // exp(gamma)
    float* dec = Gs + kChunk;             // exp(gamma_n - gamma)
    float* bG = dec + kChunk;             // beta * Gam
    float* dgam = bG + kChunk;            // d gamma
    float* rowKd = dgam + kChunk;         // rowdot(Kd, dKd)
    float* red = rowKd + kChunk;          // [32] block reduction scratch

    const Tin* qp = (const Tin*)p.q;
    const Tin* kp = (const Tin*)p.k;
    const Tin* vp = (const Tin*)p.v;
    const Tin* dop = (const Tin*)b.dout;
    const int64_t ch = (int64_t)c * p.Hv + h;
    const float* Uc = U + ch * kChunk * dv;
    const float* dUc = dU + ch * kChunk * dv;
    const float* H = Hc + ch * dk * dv;
    const float* dH = dHc + ch * dk * dv;
    auto dO = [&](int r, int j) { return to_f(dop[((int64_t)(t0 + r) * p.Hv + h) * dv + j]); };
    auto Vv = [&](int r, int j) { return to_f(vp[((int64_t)(t0 + r) * p.Hv + h) * dv + j]); };

    // S1: chunk inputs and gates
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        const int64_t off = ((int64_t)(t0 + r) * p.Hk + hk) * dk + i;
        Qs[idx] = r < n ? to_f(qp[off]) : 0.f;
        Ks[idx] = r < n ? to_f(kp[off]) : 0.f;
    }
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        bs[r] = r < n ? gate_beta(p.beta[(int64_t)(t0 + r) * p.Hv + h], p.gate_logits) : 0.f;
        gs[r] = gam[ch * kChunk + r];
        dgam[r] = 0.f;
    }
    __syncthreads();
    if (p.qk_norm) {  // raw q and k rows: normalised before use
        l2norm_rows_smem(Qs, kChunk, dk);
        l2norm_rows_smem(Ks, kChunk, dk);
        __syncthreads();
    }
    const float gl = gs[kChunk - 1];
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        Gs[r] = expf(gs[r]);
        dec[r] = expf(gl - gs[r]);
        bG[r] = bs[r] * Gs[r];
    }
    // S2: K K^T o E (strict) and P (inclusive)
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float ke = 0.f, pv = 0.f;
        if (s <= r && r < n) {
            float dkk = 0.f, dqk = 0.f;
            for (int i = 0; i < dk; ++i) {
                dkk += Ks[r * dk + i] * Ks[s * dk + i];
                dqk += Qs[r * dk + i] * Ks[s * dk + i];
            }
            const float e = expf(gs[r] - gs[s]);
            if (s < r) ke = dkk * e;
            pv = dqk * e;
        }
        KE[idx] = ke;
        Pb[idx] = pv;
    }
    __syncthreads();
    // S3: T = (I + A)^-1 (A = diag(beta) KE); dP = lower-incl(dO U^T)
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
                for (int j = col; j < r; ++j) s += bs[r] * KE[r * kChunk + j] * Tm[j * kChunk + col];
                val = -s;
            }
            Tm[r * kChunk + col] = val;
        }
    }
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float v = 0.f;
        if (s <= r && r < n)
            for (int j = 0; j < dv; ++j) v += dO(r, j) * Uc[s * dv + j];
        dP[idx] = v;
    }
    __syncthreads();
    // S4: dgamma += rowsum - colsum (dP o P); then dP <- dP o E
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        float acc = 0.f;
        for (int s = 0; s < kChunk; ++s)
            acc += dP[r * kChunk + s] * Pb[r * kChunk + s] - dP[s * kChunk + r] * Pb[s * kChunk + r];
        dgam[r] += acc;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        if (s <= r && r < n) dP[idx] *= expf(gs[r] - gs[s]);
    }
    // S5: dW = -dU H^T
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        float acc = 0.f;
        if (r < n)
            for (int j = 0; j < dv; ++j) acc -= dUc[r * dv + j] * H[(int64_t)i * dv + j];
        Wb[idx] = acc;
    }
    __syncthreads();
    // S6: dT (strictly lower part is all that reaches dA)
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float v = 0.f;
        if (s < r && r < n) {
            float a = 0.f;
            for (int i = 0; i < dk; ++i) a += Wb[r * dk + i] * Ks[s * dk + i];
            float u = 0.f;
            for (int j = 0; j < dv; ++j) u += dUc[r * dv + j] * Vv(s, j);
            v = bG[s] * a + bs[s] * u;
        }
        dA[idx] = v;
    }
    __syncthreads();
    // S7: Y = dT T^T  (into Pb)
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float v = 0.f;
        for (int bb = 0; bb <= s && bb < r; ++bb) v += dA[r * kChunk + bb] * Tm[s * kChunk + bb];
        Pb[idx] = v;
    }
    __syncthreads();
    // S8: dA = strictly-lower(-T^T Y)
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float v = 0.f;
        if (s < r && r < n)
            for (int a = r; a < kChunk; ++a) v -= Tm[a * kChunk + r] * Pb[a * kChunk + s];
        dA[idx] = v;
    }
    // S9: T^T dW
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
        const int r = idx / dk, i = idx % dk;
        float acc = 0.f;
        for (int a = r; a < kChunk; ++a) acc += Tm[a * kChunk + r] * Wb[a * dk + i];
        TW[idx] = acc;
    }
    __syncthreads();
    // S10: per row: dv, dbeta, and the T / A parts of dgamma
    Tin* dvp = (Tin*)b.dv;
    for (int r = warp; r < n; r += nwarps) {
        float acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, acc4 = 0.f;
        for (int j = lane; j < dv; j += 32) {
            float tdu = 0.f;
            for (int a = r; a < n; ++a) tdu += Tm[a * kChunk + r] * dUc[a * dv + j];
            store_as(dvp + ((int64_t)(t0 + r) * p.Hv + h) * dv + j, bs[r] * tdu);
            acc1 += tdu * Vv(r, j);
        }
        for (int i = lane; i < dk; i += 32) acc2 += TW[r * dk + i] * Ks[r * dk + i];
        for (int s = lane; s < kChunk; s += 32) {
            acc3 += dA[r * kChunk + s] * KE[r * kChunk + s];
            acc4 += bs[r] * dA[r * kChunk + s] * KE[r * kChunk + s] -
                    bs[s] * dA[s * kChunk + r] * KE[s * kChunk + r];
        }
        acc1 = warp_sum(acc1);
        acc2 = warp_sum(acc2);
        acc3 = warp_sum(acc3);
        acc4 = warp_sum(acc4);
        if (lane == 0) {
            b.dbeta[(int64_t)(t0 + r) * p.Hv + h] = gate_beta_grad(acc1 + Gs[r] * acc2 + acc3, bs[r], p.gate_logits);
            dgam[r] += bG[r] * acc2 + acc4;
        }
    }
    __syncthreads();
    // S11: G = dA o E o beta_row (in place)
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        if (s < r && r < n) dA[idx] *= expf(gs[r] - gs[s]) * bs[r];
    }
    __syncthreads();
    // S12: per row: dq, dk and the rest of dgamma
    for (int r = warp; r < n; r += nwarps) {
        float accQ = 0.f, accK = 0.f;
        for (int i = lane; i < dk; i += 32) {
            float qs = 0.f, dkd = 0.f;
            for (int j = 0; j < dv; ++j) {
                qs += dO(r, j) * H[(int64_t)i * dv + j];
                dkd += Uc[r * dv + j] * dH[(int64_t)i * dv + j];
            }
            qs *= Gs[r];
            float dq = qs;
            for (int s = 0; s <= r; ++s) dq += dP[r * kChunk + s] * Ks[s * dk + i];
            float dkv = dec[r] * dkd + bG[r] * TW[r * dk + i];
            for (int s = r; s < n; ++s) dkv += dP[s * kChunk + r] * Qs[s * dk + i];
            for (int s = 0; s < n; ++s) dkv += (dA[r * kChunk + s] + dA[s * kChunk + r]) * Ks[s * dk + i];
            accQ += Qs[r * dk + i] * qs;
            accK += dec[r] * Ks[r * dk + i] * dkd;
            dqw[((int64_t)(t0 + r) * p.Hv + h) * dk + i] = dq;
            dkw[((int64_t)(t0 + r) * p.Hv + h) * dk + i] = dkv;
        }
        accQ = warp_sum(accQ);
        accK = warp_sum(accK);
        if (lane == 0) {
            dgam[r] += accQ - accK;
            rowKd[r] = accK;
        }
    }
    // <dH, H>
    float hh = 0.f;
    for (int idx = threadIdx.x; idx < dk * dv; idx += blockDim.x) hh += dH[idx] * H[idx];
    hh = warp_sum(hh);
    if (lane == 0) red[warp] = hh;
    __syncthreads();
    if (threadIdx.x == 0) {
        float tot = 0.f;
        for (int w = 0; w < nwarps; ++w) tot += red[w];
        float kd = 0.f;
        for (int r = 0; r < n; ++r) kd += rowKd[r];
        dgam[n - 1] += kd + expf(gl) * tot;
        float run = 0.f;
        for (int r = n - 1; r >= 0; --r) {  // dg = reverse in-chunk cumsum
            run += dgam[r];
            b.dg[(int64_t)(t0 + r) * p.Hv + h] =
                gate_g_grad(run, p.gate_logits ? p.g[(int64_t)(t0 + r) * p.Hv + h] : 0.f, p.gate_logits);
        }
    }
}

// dq/dk: sum the per-value-head gradients of each q/k head's group.
template <typename Tin>
__global__ void simt_bwd_reduce_kernel(BwdProblem b, const float* dqw, const float* dkw) {
    const Problem& p = b.f;
    const int64_t total = p.T_total * p.Hk * p.dk;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(idx % p.dk);
        const int64_t th = idx / p.dk;
        const int hk = (int)(th % p.Hk);
        const int64_t t = th / p.Hk;
        float sq = 0.f, sk = 0.f;
        for (int gg = 0; gg < p.group; ++gg) {
            const int64_t src = (t * p.Hv + hk * p.group + gg) * p.dk + i;
            sq += dqw[src];
            sk += dkw[src];
        }
        store_as((Tin*)b.dq + idx, sq);
        store_as((Tin*)b.dk + idx, sk);
    }
}

// GDN_FLAG_QK_L2NORM: one warp per (token, q/k head) row sums the per-value-head gradients of
// the normalised row y = x / max(|x|, eps) over the group, then takes them back to the raw row x:
// dx = (dy - y (y . dy)) / max(|x|, eps), or dy / eps where the clamp holds (dk <= 128: four
// elements per lane).
template <typename Tin>
__global__ void simt_bwd_reduce_l2norm_kernel(BwdProblem b, const float* dqw, const float* dkw) {
    const Problem& p = b.f;
    const int lane = threadIdx.x & 31;
    const int64_t rows = p.T_total * p.Hk;
    const int64_t wstride = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; row < rows; row += wstride) {
        const int hk = (int)(row % p.Hk);
        const int64_t t = row / p.Hk;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const float* w = which ? dkw : dqw;
            const Tin* x = (const Tin*)(which ? p.k : p.q) + row * p.dk;
            Tin* out = (Tin*)(which ? b.dk : b.dq) + row * p.dk;
            float dy[4], xv[4], ss = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = lane + 32 * e;
                float acc = 0.f, xi = 0.f;
                if (i < p.dk) {
                    for (int gg = 0; gg < p.group; ++gg) acc += w[(t * p.Hv + hk * p.group + gg) * p.dk + i];
                    xi = to_f(x[i]);
                }
                dy[e] = acc;
                xv[e] = xi;
                ss += xi * xi;
            }
            ss = warp_sum(ss);
            const float nrm = sqrtf(ss), inv = 1.f / fmaxf(nrm, kL2Eps);
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) dot += xv[e] * inv * dy[e];
            dot = warp_sum(dot);
            const bool clamped = !(nrm > kL2Eps);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = lane + 32 * e;
                if (i < p.dk) store_as(out + i, clamped ? dy[e] * inv : (dy[e] - xv[e] * inv * dot) * inv);
            }
        }
    }
}

template <typename Tin>
static gdn_status launch_reduce_t(const BwdProblem& b, const float* dqw, const float* dkw, cudaStream_t s) {
    const Problem& p = b.f;
    if (p.qk_norm) {
        const int64_t rows = p.T_total * p.Hk;
        const int blocks = (int)std::min<int64_t>((rows + 7) / 8, 148 * 16);  // 8 rows per block
        simt_bwd_reduce_l2norm_kernel<Tin><<<blocks, 256, 0, s>>>(b, dqw, dkw);
    } else {
        const int64_t total = p.T_total * p.Hk * p.dk;
        const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
        simt_bwd_reduce_kernel<Tin><<<blocks, 256, 0, s>>>(b, dqw, dkw);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename K>
static gdn_status set_smem_b(K kernel, size_t bytes) {
    if (bytes > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
            cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

template <typename Tin>
static gdn_status launch_bwd_typed(const BwdPlan& plan, char* ws, cudaStream_t s) {
    const BwdProblem& b = plan.b;
    const Problem& p = b.f;
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
    float* dHc = (float*)(ws + plan.off_dHc);
    float* dU = (float*)(ws + plan.off_dU);
    float* dqw = (float*)(ws + plan.off_dqw);
    float* dkw = (float*)(ws + plan.off_dkw);
    gdn_status st = launch_chunk_table(p, ct, s);
    if (st) return st;
    if (nc > 0) {
        if ((st = launch_simt_wy(p, ct, W, U, gam, s))) return st;
        if ((st = launch_simt_state(p, ct, W, U, gam, Hc, nullptr, s))) return st;
    }
    {
        const size_t smem = sizeof(float) * (2 * kChunk * p.dk + kChunk * kChunk + p.dk * kSliceB +
                                             2 * kChunk * kSliceB + kChunk);
        if (set_smem_b(simt_bwd_dstate_kernel<Tin>, smem)) return GDN_ERR_CUDA;
        dim3 grid(p.N, p.Hv, (p.dv + kSliceB - 1) / kSliceB);
        simt_bwd_dstate_kernel<Tin><<<grid, 256, smem, s>>>(b, ct, W, gam, dHc, dU);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (nc > 0) {
        const size_t smem =
            sizeof(float) * (4 * kChunk * p.dk + 5 * kChunk * kChunk + 7 * kChunk + 32);
        if (set_smem_b(simt_bwd_chunk_kernel<Tin>, smem)) return GDN_ERR_CUDA;
        dim3 grid((unsigned)nc, p.Hv);
        simt_bwd_chunk_kernel<Tin><<<grid, 256, smem, s>>>(b, ct, U, gam, Hc, dHc, dU, dqw, dkw);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
        const gdn_status st = launch_reduce_t<Tin>(b, dqw, dkw, s);
        if (st) return st;
    }
    return GDN_OK;
}

gdn_status launch_bwd_reduce(const BwdProblem& b, const float* dqw, const float* dkw, cudaStream_t s) {
    return b.f.dtype == GDN_BF16 ? launch_reduce_t<__nv_bfloat16>(b, dqw, dkw, s)
                                 : launch_reduce_t<float>(b, dqw, dkw, s);
}

gdn_status launch_bwd_simt(const BwdPlan& plan, char* ws, cudaStream_t s) {
    return plan.b.f.dtype == GDN_BF16 ? launch_bwd_typed<__nv_bfloat16>(plan, ws, s)
                                      : launch_bwd_typed<float>(plan, ws, s);
}

}  // namespace gdn
