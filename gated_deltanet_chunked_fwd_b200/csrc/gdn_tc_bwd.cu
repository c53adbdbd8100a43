// gdn_tc_bwd.cu -- tensor-core backward of the chunked gated delta rule (bf16, dk = dv = 128,
// sm_100a).  The backward of the GDN layer (FlashQLA pages: dothoosh.com article, opening
// paragraph, "backward pass"; news.hamidun.com page, "large-scale pretraining" scenario).
//
// One CTA per (sequence, value head), 128 threads (thread i <-> TMEM lane i <-> MMA row i).
// Phase 1 replays the forward chain (as the fused forward kernel does) and saves, per chunk,
// the bf16 entry state H^T and the bf16 T = (I + A)^-1 as ready-to-use 128-byte-swizzled
// shared-memory images in the workspace.  Phase 2 walks the chunks backwards with the state
// adjoint dH (fp32, TMEM) and, per chunk (notation of gdn_internal.cuh; E, Gam, dec, beta
// from the gates; Kb = diag(beta Gam) K):
//   U^T  = Ut^T - H^T W^T                         (recomputed, MMAs)
//   dU^T = dO^T P + (dH^T K^T) diag(dec)
//   TdU^T = dU^T T            (TdU = T^T dU;  dv = diag(beta) TdU)
//   dH  <- Gam_n dH + (diag(Gam) Q)^T dO - W^T dU    (next chunk's exit adjoint)
//   [dP ; dA'] = [dO ; TdU] U^T,  dP masked lower-incl,  dA = -strictly-lower(dA')
//                (dA = -strictly-lower(T^T dT T^T) with dT = dU U^T (I + A)^T)
//   dq^T = Gam o (H dO^T) + K^T (dP o E)^T
//   dk^T = Q^T (dP o E) + K^T (G + G^T)^T + dec o (dH U^T) + beta Gam o (-(H TdU^T))
//          with G = dA o E o beta_row
//   dbeta, dgamma: row sums of the same products (cross-lane reductions); dg = reverse
//   cumsum of dgamma.  dS0 is the final dH.
// Every product is an M = 128 tcgen05.mma (M = a head dimension, or the stacked 128 rows of
// [dO ; TdU]); A operands come from shared memory (either major) or TMEM (dH^T, dU^T bf16).
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kNT = 128;
constexpr int kTmemColsB = 512;
// TMEM columns (lane = MMA row)
constexpr uint32_t cH = 0;     // phase 1: H^T fp32; phase 2: dH^T fp32          [0, 128)
constexpr uint32_t cHb = 128;  // phase 2: bf16 dH^T (A operand)                  [128, 192)
constexpr uint32_t cR1 = 192;  // Q K^T / K K^T, later dk^T (main part)
constexpr uint32_t cR2 = 256;  // W^T, later TdU^T, later dKd^T
constexpr uint32_t cR3 = 320;  // Ut^T -> U^T, later [dP ; dA'], later K^T (dP o E)^T
constexpr uint32_t cR4 = 384;  // dO^T P, later H dO^T
constexpr uint32_t cR5 = 448;  // dH^T K^T, then bf16 dU^T (cols 0..31), later TdW^T

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t bQK = 0;        // 32 KB [dk atom][q rows 0-63 | k rows 64-127][128 B]
constexpr uint32_t bV = 32768;     // 16 KB [dv atom][64 rows][128 B]; phase 2: fp32 G [64][64]
constexpr uint32_t bDO = 49152;    // 32 KB [dv atom][do rows 0-63 | TdU rows 64-127][128 B]
constexpr uint32_t bHt = 81920;    // 32 KB bf16 H^T [dk atom][128 dv rows][128 B]
constexpr uint32_t bT = 114688;    // 8 KB  T [64 rows s][64 r]; later S = G + G^T [s][j]
constexpr uint32_t bBw = 122880;   // 8 KB  T diag(beta Gam) | phase 1: fp32 A (16 KB over Bw+Bu)
constexpr uint32_t bBu = 131072;   // 8 KB  T diag(beta)     | phase 2: diag(Gam) Q [atom][64][128]
constexpr uint32_t bP = 139264;    // 8 KB  P [64 r][64 s]; later dP o E
constexpr uint32_t bWt = 147456;   // 16 KB -W^T [128 dk rows][64 s]; later -TdU^T [128 dv rows][64 r]
constexpr uint32_t bUt = 163840;   // 16 KB phase 1: U^T diag(dec); phase 2: U^T [128 dv rows][64 s]
constexpr uint32_t bDHt = 180224;  // 32 KB phase 2: bf16 dH^T; phase 1: fp32 T [64][68] + scratch
constexpr uint32_t bM = bDHt;
constexpr uint32_t bYs = bDHt + 64 * kLd * 4;
constexpr uint32_t bVec = 212992;  // per-token vectors (8 x 64 floats)
constexpr uint32_t bRed = bVec + 2048;  // reductions [4][64] floats + accumulators [4][64]
constexpr uint32_t bBar = bRed + 2048;
constexpr uint32_t kSmemB = bBar + 64 + 1024;
static_assert(bYs + 3 * 16 * kLdY * 4 <= bDHt + 32768, "phase-1 solve scratch too large");

constexpr uint32_t kHImg = 32768;  // bytes of one saved H^T image
constexpr uint32_t kTImg = 8192;   // bytes of one saved T image

struct TcBwdArgs {
    BwdProblem b;
    uint8_t* himg;   // [global chunk][Hv] H^T images
    uint8_t* timg;   // [global chunk][Hv] T images
    float* dqw;      // [T_total][Hv][dk] per-value-head dq
    float* dkw;      // [T_total][Hv][dk] per-value-head dk
};

// Reduce-scatter over a warp: lane L ends with the warp-sums of indices L*(N/32) .. +N/32-1
// in v[0 .. N/32-1].
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float* v, int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = N >> (step + 1);
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float send = upper ? v[j] : v[j + half];
            const float keep = upper ? v[j + half] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

__device__ __forceinline__ float bf(const uint8_t* tile, int row, int col) {  // bf16 element of a swizzled tile
    const uint8_t* p = tile + sw128_off(row, (col & 63) >> 3) + (col & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

__global__ void __launch_bounds__(kNT, 1)
    gdn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const TcBwdArgs args) {
    const BwdProblem& b = args.b;
    const Problem& p = b.f;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* vbeta = (float*)(sm + bVec);
    float* vGam = vbeta + 64;
    float* vbG = vbeta + 128;
    float* vdec = vbeta + 192;
    float* va = vbeta + 256;
    float* vb = vbeta + 320;
    float* vgam = vbeta + 384;
    float* red = (float*)(sm + bRed);        // [4][64]
    float* acc_g = red + 256;                // dgamma accumulator [64]
    float* acc_b = red + 320;                // dbeta accumulator [64]
    float* acc_s = red + 384;                // scalars
    uint64_t* bar_ld = (uint64_t*)(sm + bBar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* tmem_slot = (uint32_t*)(bar_mma + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hv = p.Hv, dk = 128, dv = 128;
    const int h = blockIdx.x % Hv, n = blockIdx.x / Hv, hk = h / p.group;

    // sequence bounds and its first global chunk index
    int64_t bos, len;
    int cbase;
    if (!p.cu) {
        bos = (int64_t)n * p.T;
        len = p.T;
        cbase = n * ((p.T + kChunk - 1) / kChunk);
    } else {
        bos = p.cu[n];
        len = max((int64_t)0, (int64_t)p.cu[n + 1] - bos);
        int acc = 0;  // chunks of the sequences before n (warp-cooperative)
        for (int m0 = 0; m0 < n; m0 += 32) {
            const int m = m0 + lane;
            int c = 0;
            if (m < n) c = (int)(((int64_t)p.cu[m + 1] - p.cu[m] + kChunk - 1) / kChunk);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            acc += c;
        }
        cbase = acc;
    }
    const int nck = (int)((len + kChunk - 1) / kChunk);

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemColsB);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t sb = smem_u32(sm);
    const int m = tid;  // TMEM lane / head-dimension index owned by this thread
    uint32_t ph_ld = 0, ph_mma = 0;
    bool ok = true;

    const uint32_t id_kk64 = idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mk64 = idesc_bf16(128, 64, 1, 0);
    const uint32_t id_km64 = idesc_bf16(128, 64, 0, 1);
    const uint32_t id_mm64 = idesc_bf16(128, 64, 1, 1);
    const uint32_t id_km128 = idesc_bf16(128, 128, 0, 1);
    const uint32_t id_mm128 = idesc_bf16(128, 128, 1, 1);
    const uint32_t id_kk128 = idesc_bf16(128, 128, 0, 0);
    const float LOG2E = 1.4426950408889634f;

    auto mma_sync_wait = [&]() -> bool {
        if (tid == 0) mma_commit(bar_mma);
        const bool r = __syncthreads_and(mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
        tc_fence_after();
        return r;
    };
    // gates of chunk c: beta, gamma (cumsum), Gam, beta Gam, decay to the chunk end, E factors
    auto gates = [&](int c, int lc) -> bool {
        const int64_t t0 = bos + (int64_t)c * kChunk;
        float gr = 0.f, gm = 0.f;
        if (tid < 64) {
            float x = tid < lc ? p.g[(t0 + tid) * Hv + h] : 0.f;
            const float bt = tid < lc ? p.beta[(t0 + tid) * Hv + h] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            vbeta[tid] = bt;
            vgam[tid] = x;
        }
        __syncthreads();
        if (tid < 64) {
            gr = vgam[tid] + (tid >= 32 ? vgam[31] : 0.f);
            gm = vgam[31];
            const float gl = vgam[63] + vgam[31];
            const float eg = expf(gr);
            vGam[tid] = eg;
            vbG[tid] = vbeta[tid] * eg;
            vdec[tid] = expf(gl - gr);
        }
        const bool fac = !__syncthreads_or(tid < 64 && !(fabsf(gr - gm) < 80.f));
        if (tid < 64) {
            va[tid] = fac ? expf(gr - gm) : gr * LOG2E;
            vb[tid] = fac ? expf(gm - gr) : gr * LOG2E;
        }
        __syncthreads();
        return fac;
    };
    auto Efac = [&](bool fac, int r, int s) -> float {
        return fac ? va[r] * vb[s] : exp2f(va[r] - vb[s]);
    };
    auto mma1 = [&]() {  // [Q;K] K^T -> R1
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + cR1, desc_sw128(sb + bQK + koff, 16, 1024),
                            desc_sw128(sb + bQK + 8192 + koff, 16, 1024), id_kk64, j > 0);
            }
        }
    };
    auto load_qkv = [&](int c, bool with_do, bool with_imgs) {
        if (tid == 0) {
            const int t0 = (int)(bos + (int64_t)c * kChunk);
            uint32_t bytes = 49152 + (with_do ? 16384 : 0) + (with_imgs ? kHImg + kTImg : 0);
            mbar_arrive_expect_tx(bar_ld, bytes);
            for (int a = 0; a < 2; ++a) {
                tma_load_3d(sm + bQK + a * 16384, &tm_q, bar_ld, 64 * a, hk, t0);
                tma_load_3d(sm + bQK + a * 16384 + 8192, &tm_k, bar_ld, 64 * a, hk, t0);
                tma_load_3d(sm + bV + a * 8192, &tm_v, bar_ld, 64 * a, h, t0);
                if (with_do) tma_load_3d(sm + bDO + a * 16384, &tm_do, bar_ld, 64 * a, h, t0);
            }
            if (with_imgs) {
                const int64_t gi = (int64_t)(cbase + c) * Hv + h;
                bulk_load(sm + bHt, args.himg + gi * kHImg, kHImg, bar_ld);
                bulk_load(sm + bT, args.timg + gi * kTImg, kTImg, bar_ld);
            }
        }
    };

    // ===================== phase 1: forward replay, saving H^T and T per chunk =====================
    {
        const float* s0 = p.S0 ? p.S0 + ((int64_t)n * Hv + h) * dk * dv : nullptr;
        float v[64];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = s0 ? s0[(int64_t)(64 * a + e) * dv + m] : 0.f;
            tmem_st64(tl + cH + 64 * a, v);
            store_row32(sm + bHt + a * 16384, m, 0, v);
            store_row32(sm + bHt + a * 16384, m, 4, v + 32);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    for (int c = 0; c < nck && ok; ++c) {
        const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
        const int64_t gi = (int64_t)(cbase + c) * Hv + h;
        load_qkv(c, false, false);
        const bool fac = gates(c, lc);
        ok = __syncthreads_and(mbar_wait(bar_ld, ph_ld));
        ph_ld ^= 1;
        if (!ok) break;
        mma1();
        // save the entry state image while MMA1 runs
        {
            const uint4* src = reinterpret_cast<const uint4*>(sm + bHt);
            uint4* dst = reinterpret_cast<uint4*>(args.himg + gi * kHImg);
            for (int i = tid; i < (int)(kHImg / 16); i += kNT) dst[i] = src[i];
        }
        if (!(ok = mma_sync_wait())) break;
        // A (rows 64..127 of R1) -> fp32, swizzled, over Bw/Bu
        if (tid >= 64) {
            const int r = tid - 64;
            float v[64];
            tmem_ld64(tl + cR1, v);
            float* As = (float*)(sm + bBw);
            const float br = vbeta[r];
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                float4 w;
                float* wp = &w.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = 4 * c4 + e;
                    wp[e] = (s < r && r < lc) ? br * v[s] * Efac(fac, r, s) : 0.f;
                }
                *reinterpret_cast<float4*>(As + as_idx(r, 4 * c4)) = w;
            }
        }
        tc_fence_before();
        __syncthreads();
        {
            const float* As = (const float*)(sm + bBw);
            float* M = (float*)(sm + bM);
            float* Ys = (float*)(sm + bYs);
            solve_diag(As, M, tid);
            __syncthreads();
            solve_level_Y<1, kNT>(As, M, Ys, tid);
            __syncthreads();
            solve_level_T<1, kNT>(M, Ys, tid);
            __syncthreads();
            solve_level_Y<2, kNT>(As, M, Ys, tid);
            __syncthreads();
            solve_level_T<2, kNT>(M, Ys, tid);
            __syncthreads();
            solve_level_Y<3, kNT>(As, M, Ys, tid);
            __syncthreads();
            solve_level_T<3, kNT>(M, Ys, tid);
            __syncthreads();
            // Bw = T diag(beta Gam), Bu = T diag(beta) into smem; the T image to the workspace
            const int nrow = tid >> 1, hf = tid & 1;
            float vw[32], vu[32], vt[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = 32 * hf + e;
                const float t = (s <= nrow) ? M[nrow * kLd + s] : 0.f;
                vt[e] = t;
                vw[e] = t * vbG[s];
                vu[e] = t * vbeta[s];
            }
            __syncthreads();  // As (over Bw/Bu) is no longer read
            store_row32(sm + bBw, nrow, 4 * hf, vw);
            store_row32(sm + bBu, nrow, 4 * hf, vu);
            uint8_t* timg = args.timg + gi * kTImg;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                *reinterpret_cast<uint4*>(timg + sw128_off(nrow, 4 * hf + cc)) = pack8(vt + 8 * cc);
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {  // W^T = K^T Bw^T (R2);  Ut^T = V^T Bu^T (R3)
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mma_bf16_ss(tmem + cR2, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                            desc_sw128(sb + bBw + j * 32, 16, 1024), id_mk64, j > 0);
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bV + j * 2048, 8192, 1024),
                            desc_sw128(sb + bBu + j * 32, 16, 1024), id_mk64, j > 0);
            }
        }
        if (!(ok = mma_sync_wait())) break;
        {  // -W^T -> Wt
            float v[64];
            tmem_ld64(tl + cR2, v);
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = -v[e];
            store_row32(sm + bWt, m, 0, v);
            store_row32(sm + bWt, m, 4, v + 32);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // U^T = Ut^T + H^T (-W^T)
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bHt + koff, 16, 1024),
                            desc_sw128(sb + bWt + j * 2048, 8192, 1024), id_km64, 1);
            }
        }
        if (!(ok = mma_sync_wait())) break;
        {  // U^T diag(dec) -> Ut;  H^T <- Gam_n H^T
            float v[64];
            tmem_ld64(tl + cR3, v);
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] *= vdec[e];
            store_row32(sm + bUt, m, 0, v);
            store_row32(sm + bUt, m, 4, v + 32);
            const float Gn = vGam[63];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + cH + 64 * a, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] *= Gn;
                tmem_st64(tl + cH + 64 * a, v);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // H^T += (U^T diag(dec)) K
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_bf16_ss(tmem + cH, desc_sw128(sb + bUt + j * 32, 16, 1024),
                            desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024), id_km128, 1);
        }
        if (!(ok = mma_sync_wait())) break;
        {  // bf16 copy of the new state (next chunk's A operand and saved image)
            float v[64];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + cH + 64 * a, v);
                store_row32(sm + bHt + a * 16384, m, 0, v);
                store_row32(sm + bHt + a * 16384, m, 4, v + 32);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    // ===================== phase 2: reverse walk with the state adjoint =====================
    if (ok) {  // dH^T <- dS_T
        const float* dst = b.dST ? b.dST + ((int64_t)n * Hv + h) * dk * dv : nullptr;
        float v[64];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = dst ? dst[(int64_t)(64 * a + e) * dv + m] : 0.f;
            tmem_st64(tl + cH + 64 * a, v);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    for (int c = nck - 1; c >= 0 && ok; --c) {
        const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
        const int64_t t0 = bos + (int64_t)c * kChunk;
        // bf16 copies of the exit adjoint dH_c: TMEM (A operand) and smem (MN-major A of dKd)
        {
            float v[64];
            uint32_t w[32];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + cH + 64 * a, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
                tmem_st32u(tl + cHb + 32 * a, w);
                store_row32(sm + bDHt + a * 16384, m, 0, v);
                store_row32(sm + bDHt + a * 16384, m, 4, v + 32);
            }
        }
        if (tid < 64) {
            acc_g[tid] = 0.f;
            acc_b[tid] = 0.f;
        }
        if (tid < 8) acc_s[tid] = 0.f;
        load_qkv(c, true, true);
        const bool fac = gates(c, lc);
        ok = __syncthreads_and(mbar_wait(bar_ld, ph_ld));
        ph_ld ^= 1;
        if (!ok) break;
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        mma1();
        if (!(ok = mma_sync_wait())) break;
        // P (rows 0..63) -> smem; Bw, Bu from the T image
        if (tid < 64) {
            const int r = tid;
            float v[64];
            tmem_ld64(tl + cR1, v);
#pragma unroll
            for (int s = 0; s < 64; ++s) v[s] = (s <= r && r < lc) ? v[s] * Efac(fac, r, s) : 0.f;
            store_row32(sm + bP, r, 0, v);
            store_row32(sm + bP, r, 4, v + 32);
        }
        {
            const int nrow = tid >> 1, hf = tid & 1;
            float vw[32], vu[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = 32 * hf + e;
                const float t = bf(sm + bT, nrow, s);
                vw[e] = t * vbG[s];
                vu[e] = t * vbeta[s];
            }
            store_row32(sm + bBw, nrow, 4 * hf, vw);
            store_row32(sm + bBu, nrow, 4 * hf, vu);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // W^T (R2), Ut^T (R3)
                mma_bf16_ss(tmem + cR2, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                            desc_sw128(sb + bBw + j * 32, 16, 1024), id_mk64, j > 0);
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bV + j * 2048, 8192, 1024),
                            desc_sw128(sb + bBu + j * 32, 16, 1024), id_mk64, j > 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)  // dO^T P (R4): A = dO^T MN-major, B = P MN-major (N = s)
                mma_bf16_ss(tmem + cR4, desc_sw128(sb + bDO + j * 2048, 16384, 1024),
                            desc_sw128(sb + bP + j * 2048, 8192, 1024), id_mm64, j > 0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // dH^T K^T (R5): A = bf16 dH^T (TMEM), B = K rows
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ts(tmem + cR5, tmem + cHb + 8 * j, desc_sw128(sb + bQK + 8192 + koff, 16, 1024),
                            id_kk64, j > 0);
            }
        }
        if (!(ok = mma_sync_wait())) break;
        {  // -W^T -> Wt;  Q rows * Gam -> Qg (over Bw/Bu);  dU^T -> bf16 (R5 cols 0..31);
           // <dH_c, H_c>, then dH^T <- Gam_n dH^T
            float v[64];
            tmem_ld64(tl + cR2, v);
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = -v[e];
            store_row32(sm + bWt, m, 0, v);
            store_row32(sm + bWt, m, 4, v + 32);
            {
                // rows past the sequence end hold the next sequence's q and dO: zero them here
                const int r = m >> 1, a = m & 1;
                const float gmul = r < lc ? vGam[r] : 0.f;
                const uint4* src = reinterpret_cast<const uint4*>(sm + bQK + a * 16384 + r * 128);
                uint4* dst = reinterpret_cast<uint4*>(sm + bBw + a * 8192 + r * 128);
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) {
                    const int c8 = (i8 + r) & 7;
                    uint4 u = src[c8];
                    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 f = __bfloat1622float2(b2[e]);
                        b2[e] = __floats2bfloat162_rn(f.x * gmul, f.y * gmul);
                    }
                    dst[c8] = u;  // same swizzle position: row r keeps its chunk permutation
                }
            }
            float w64[64];
            tmem_ld64x2(tl + cR4, v, tl + cR5, w64);
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
                w[e] = pack_bf16(v[2 * e] + vdec[2 * e] * w64[2 * e], v[2 * e + 1] + vdec[2 * e + 1] * w64[2 * e + 1]);
            tmem_st32u(tl + cR5, w);
            float dhh = 0.f;
            const float Gn = vGam[63];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + cH + 64 * a, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    dhh += v[e] * bf(sm + bHt + a * 16384, m, e);
                    v[e] *= Gn;
                }
                tmem_st64(tl + cH + 64 * a, v);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dhh += __shfl_xor_sync(0xffffffffu, dhh, o);
            if (lane == 0) atomicAdd(&acc_s[0], dhh);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // U^T = Ut^T + H^T (-W^T)   (R3)
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bHt + koff, 16, 1024),
                            desc_sw128(sb + bWt + j * 2048, 8192, 1024), id_km64, 1);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)  // TdU^T = dU^T T   (R2): B = T MN-major (N = r)
                mma_bf16_ts(tmem + cR2, tmem + cR5 + 8 * j, desc_sw128(sb + bT + j * 2048, 8192, 1024),
                            id_km64, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)  // dH^T += dO^T Qg   (B = Qg MN-major, N = dk)
                mma_bf16_ss(tmem + cH, desc_sw128(sb + bDO + j * 2048, 16384, 1024),
                            desc_sw128(sb + bBw + j * 2048, 8192, 1024), id_mm128, 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)  // dH^T += dU^T (-W)  (B = -W^T rows, K-major)
                mma_bf16_ts(tmem + cH, tmem + cR5 + 8 * j, desc_sw128(sb + bWt + j * 32, 16, 1024),
                            id_kk128, 1);
        }
        if (!(ok = mma_sync_wait())) break;
        {  // U^T -> Ut;  TdU: dv out, rows 64..127 of the dO tile, -TdU^T -> Wt, dbeta part
            float v[64];
            tmem_ld64(tl + cR3, v);
            store_row32(sm + bUt, m, 0, v);
            store_row32(sm + bUt, m, 4, v + 32);
            tmem_ld64(tl + cR2, v);
            __nv_bfloat16* dvp = (__nv_bfloat16*)b.dv + (t0 * Hv + h) * dv + m;
            float bvals[64];
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                if (r < lc) dvp[(int64_t)r * Hv * dv] = __float2bfloat16_rn(vbeta[r] * v[r]);
                bvals[r] = v[r] * bf(sm + bV + (m >> 6) * 8192, r, m & 63);  // TdU[r][m] v[r][m]
                // TdU row r of the stacked [dO ; TdU] tile: element (64 + r, m)
                *reinterpret_cast<__nv_bfloat16*>(sm + bDO + (m >> 6) * 16384 + sw128_off(64 + r, (m & 63) >> 3) +
                                                  (m & 7) * 2) = __float2bfloat16_rn(v[r]);
            }
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = -v[e];
            store_row32(sm + bWt, m, 0, v);
            store_row32(sm + bWt, m, 4, v + 32);
            warp_reduce_scatter<64>(bvals, lane);
            red[warp * 64 + 2 * lane] = bvals[0];
            red[warp * 64 + 2 * lane + 1] = bvals[1];
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid < 64) acc_b[tid] += red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // [dP ; dA'] = [dO ; TdU] U^T   (R3): B = U^T MN-major
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bDO + koff, 16, 1024),
                            desc_sw128(sb + bUt + j * 2048, 8192, 1024), id_km64, j > 0);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // H dO^T (R4): A = H (MN-major view of H^T), B = dO rows
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + cR4, desc_sw128(sb + bHt + j * 2048, 16384, 1024),
                            desc_sw128(sb + bDO + koff, 16, 1024), id_mk64, j > 0);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)  // TdW^T = H (-TdU^T)^T... = -H TdU^T (R5): B = -TdU^T MN-major
                mma_bf16_ss(tmem + cR5, desc_sw128(sb + bHt + j * 2048, 16384, 1024),
                            desc_sw128(sb + bWt + j * 2048, 8192, 1024), id_mm64, j > 0);
#pragma unroll
            for (int j = 0; j < 8; ++j)  // dKd^T = dH U^T (R2): A = dH (MN-major view of dH^T)
                mma_bf16_ss(tmem + cR2, desc_sw128(sb + bDHt + j * 2048, 16384, 1024),
                            desc_sw128(sb + bUt + j * 2048, 8192, 1024), id_mm64, j > 0);
        }
        if (!(ok = mma_sync_wait())) break;
        {  // dP (lanes 0..63) and dA (lanes 64..127) rows: dgamma / dbeta terms, dP o E, G
            const int r = tid & 63;
            float d[64], x[64];
            tmem_ld64x2(tl + cR3, d, tl + cR1, x);
            float rowsum = 0.f, bsum = 0.f;
            if (tid < 64) {
#pragma unroll
                for (int s = 0; s < 64; ++s) {
                    const bool in = (s <= r && r < lc);
                    const float E = Efac(fac, r, s);
                    const float P = in ? x[s] * E : 0.f;
                    const float dP = in ? d[s] : 0.f;
                    rowsum += dP * P;
                    x[s] = dP * P;      // column-sum term
                    d[s] = dP * E;      // dP o E
                }
                store_row32(sm + bP, r, 0, d);
                store_row32(sm + bP, r, 4, d + 32);
            } else {
                float* G = (float*)(sm + bV);
                const float br = vbeta[r];
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    float4 gw;
                    float* gp = &gw.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = 4 * c4 + e;
                        const bool in = (s < r && r < lc);
                        const float E = Efac(fac, r, s);
                        const float dA = in ? -d[s] : 0.f;
                        const float KE = x[s] * E;
                        const float A = br * KE;
                        rowsum += dA * A;
                        bsum += dA * KE;
                        x[s] = dA * A;
                        gp[e] = dA * E * br;
                    }
                    *reinterpret_cast<float4*>(G + as_idx(r, 4 * c4)) = gw;
                }
            }
            warp_reduce_scatter<64>(x, lane);
            red[warp * 64 + 2 * lane] = x[0];
            red[warp * 64 + 2 * lane + 1] = x[1];
            __syncthreads();
            // dgamma_r += rowsum (own row)  -  colsum (all rows) for both dP o P and dA o A
            if (tid < 64) acc_g[tid] += rowsum - (red[tid] + red[64 + tid]);
            __syncthreads();
            if (tid >= 64) acc_g[r] += rowsum - (red[128 + r] + red[192 + r]);
            if (tid >= 64) acc_b[r] += bsum;
        }
        __syncthreads();
        if (tid < 64) {  // S = G + G^T, row s = tid
            const int s = tid;
            const float* G = (const float*)(sm + bV);
            float v[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = G[as_idx(s, j)] + G[as_idx(j, s)];
            store_row32(sm + bT, s, 0, v);
            store_row32(sm + bT, s, 4, v + 32);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j)  // K^T (dP o E)^T (R3): A = K^T MN-major, B = dPE rows K-major
                mma_bf16_ss(tmem + cR3, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                            desc_sw128(sb + bP + j * 32, 16, 1024), id_mk64, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)  // dk^T main (R1): Q^T (dP o E) + K^T S^T
                mma_bf16_ss(tmem + cR1, desc_sw128(sb + bQK + j * 2048, 16384, 1024),
                            desc_sw128(sb + bP + j * 2048, 8192, 1024), id_mm64, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_bf16_ss(tmem + cR1, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                            desc_sw128(sb + bT + j * 32, 16, 1024), id_mk64, 1);
        }
        if (!(ok = mma_sync_wait())) break;
        {  // epilogue: thread i = dk index
            const int i = m;
            float gv[64], bv[64];
            float kdk = 0.f;
            const uint8_t* qtile = sm + bQK + (i >> 6) * 16384;
            float* dqp = args.dqw + (t0 * Hv + h) * dk + i;
            float* dkp = args.dkw + (t0 * Hv + h) * dk + i;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float a32[32], b32[32];
                tmem_ld32x2(tl + cR4 + 32 * hf, a32, tl + cR3 + 32 * hf, b32);  // H dO^T, K^T dPE^T
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int r = 32 * hf + e;
                    const float qs = vGam[r] * a32[e];  // dQs^T[i][r]
                    if (r < lc) dqp[(int64_t)r * Hv * dk] = qs + b32[e];
                    gv[r] = bf(qtile, r, i & 63) * qs;
                }
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float a32[32], b32[32], c32[32];
                tmem_ld32x2(tl + cR1 + 32 * hf, a32, tl + cR2 + 32 * hf, b32);  // dk main, dKd^T
                tmem_ld32(tl + cR5 + 32 * hf, c32);                              // TdW^T
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = 32 * hf + e;
                    const float kv = bf(qtile, 64 + s, i & 63);
                    const float dkv = a32[e] + vdec[s] * b32[e] + vbG[s] * c32[e];
                    if (s < lc) dkp[(int64_t)s * Hv * dk] = dkv;
                    const float kdterm = vdec[s] * kv * b32[e];
                    gv[s] += vbG[s] * c32[e] * kv - kdterm;
                    bv[s] = vGam[s] * c32[e] * kv;
                    kdk += kdterm;
                }
            }
            warp_reduce_scatter<64>(gv, lane);
            warp_reduce_scatter<64>(bv, lane);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kdk += __shfl_xor_sync(0xffffffffu, kdk, o);
            red[warp * 64 + 2 * lane] = gv[0];
            red[warp * 64 + 2 * lane + 1] = gv[1];
            if (lane == 0) atomicAdd(&acc_s[1], kdk);
            __syncthreads();
            if (tid < 64) acc_g[tid] += red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
            __syncthreads();
            red[warp * 64 + 2 * lane] = bv[0];
            red[warp * 64 + 2 * lane + 1] = bv[1];
            __syncthreads();
            if (tid < 64) acc_b[tid] += red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
            __syncthreads();
        }
        if (tid == 0) {  // last-row terms, then dg = reverse in-chunk cumsum of dgamma
            acc_g[lc - 1] += acc_s[1] + vGam[63] * acc_s[0];
            float run = 0.f;
            for (int r = lc - 1; r >= 0; --r) {
                run += acc_g[r];
                b.dg[(t0 + r) * Hv + h] = run;
            }
        }
        if (tid < lc) b.dbeta[(t0 + tid) * Hv + h] = acc_b[tid];
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (ok && b.dS0) {
        float* dst = b.dS0 + ((int64_t)n * Hv + h) * dk * dv + m;
        float v[64];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            tmem_ld64(tl + cH + 64 * a, v);
#pragma unroll
            for (int e = 0; e < 64; ++e) dst[(int64_t)(64 * a + e) * dv] = v[e];
        }
    }
    if (!ok && tid == 0) report(p.status, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsB);
    }
}

}  // namespace

bool tc_bwd_supported(const Problem& p) { return p.dtype == GDN_BF16 && p.dk == 128 && p.dv == 128; }

size_t tc_bwd_workspace(const Problem& p, size_t* off_himg, size_t* off_timg, size_t* off_dqw,
                        size_t* off_dkw) {
    size_t off = 0;
    *off_himg = off;
    off = align_up(off + (size_t)p.num_chunks * p.Hv * kHImg, 256);
    *off_timg = off;
    off = align_up(off + (size_t)p.num_chunks * p.Hv * kTImg, 256);
    *off_dqw = off;
    off = align_up(off + sizeof(float) * (size_t)p.T_total * p.Hv * p.dk, 256);
    *off_dkw = off;
    off = align_up(off + sizeof(float) * (size_t)p.T_total * p.Hv * p.dk, 256);
    return off;
}

gdn_status launch_bwd_tc(const BwdPlan& plan, char* ws, cudaStream_t s) {
    const BwdProblem& bp = plan.b;
    const Problem& p = bp.f;
    TcBwdArgs a;
    a.b = bp;
    size_t oh, ot, oq, ok_;
    tc_bwd_workspace(p, &oh, &ot, &oq, &ok_);
    a.himg = (uint8_t*)(ws + oh);
    a.timg = (uint8_t*)(ws + ot);
    a.dqw = (float*)(ws + oq);
    a.dkw = (float*)(ws + ok_);
    CUtensorMap mq, mk, mv, mdo;
    const int64_t Tt = std::max<int64_t>(p.T_total, 1);
    if (!make_map(&mq, p.q, Tt, p.Hk) || !make_map(&mk, p.k, Tt, p.Hk) || !make_map(&mv, p.v, Tt, p.Hv) ||
        !make_map(&mdo, bp.dout, Tt, p.Hv))
        return GDN_ERR_CUDA;
    if (cudaFuncSetAttribute(gdn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemB) !=
        cudaSuccess)
        return GDN_ERR_CUDA;
    gdn_bwd_tc_kernel<<<(unsigned)(p.N * p.Hv), kNT, kSmemB, s>>>(mq, mk, mv, mdo, a);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    if (p.T_total > 0) return launch_bwd_reduce(bp, a.dqw, a.dkw, s);
    return GDN_OK;
}

}  // namespace gdn
