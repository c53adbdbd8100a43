// gdn_tc_fwd.cu -- fused tensor-core forward of the chunked gated delta rule
// for bf16 tensors with dk = dv = 128 on sm_100a.
//
// One launch does the whole forward.  Each CTA owns one (sequence, value head,
// segment of chunks) and walks its chunks in order, keeping the fp32 state in
// TMEM; per chunk of C = 64 tokens (notation of gdn_internal.cuh):
//   gates      gamma = cumsum g, Gam, E = exp(gamma_r - gamma_s)       CUDA cores
//   MMA1       [Q;K] K^T -> Q K^T and K K^T  (M=128 rows: 64 q + 64 k)  tensor core
//   WY / UT    A = strictly-lower(diag(beta) K K^T o E),
//              T = (I + A)^-1 (16x16 diagonal blocks by substitution,
//              block merges by level)                                   CUDA cores, fp32
//   MMA_W/U    W^T = K^T (T diag(beta Gam))^T,  Ut^T = V^T (T diag(beta))^T
//   MMA_HW     U^T = Ut^T - H^T W^T  (accumulated onto Ut^T, A negated)
//   MMA_HQ/UP  O^T = Gam * (H^T Q^T) + U^T P^T,  P = lower-incl(Q K^T o E)
//   MMA_H      H^T <- Gam_n H^T + (U^T diag(exp(gamma_n - gamma))) K
// All matrices are oriented so that a 128-wide head dimension is the MMA's M
// (TMEM lane = dv or dk index), so every MMA is M = 128 with N = 64 or 128.
// Operands live in shared memory as 128-byte-swizzled tiles; q / k / v tiles
// come in by TMA (double-buffered: chunk c+1 loads while chunk c computes).
//
// Long sequences are split into segments that run on different SMs
// (gate-driven context parallelism, dothoosh.com FlashQLA article, first
// innovation): a segment that does not start its sequence starts from a zero
// state w chunks early, with w the fewest whole chunks whose summed log decay
// is <= log(eps).  While 0 <= beta |k|^2 <= 2 each token's state map has norm
// <= exp(g_t), so the truncated past contributes at most eps * |H| to the
// segment's entry state.  If the decay never reaches eps, or some warm-up
// token breaks the norm condition, the segment starts exactly from the
// sequence start (from S0) instead.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"


namespace gdn {

using namespace sm100;

namespace {

constexpr int kThreads = 256;  // 8 warps: warps w and w+4 share TMEM lane quarter w%4
constexpr int kTmemCols = 512;
// TMEM column map (lane = row of the M = 128 MMA)
constexpr uint32_t kColH = 0;     // H^T, fp32 state: lane dv, column dk   [0, 128)
constexpr uint32_t kColR1 = 128;  // Q K^T / K K^T, then W^T               [128, 192)
constexpr uint32_t kColR2 = 192;  // Ut^T, then U^T                        [192, 256)
constexpr uint32_t kColHQ = 256;  // H^T Q^T                               [256, 320)
constexpr uint32_t kColUP = 320;  // U^T P^T                               [320, 384)

// shared memory carve-up (bytes from a 1024-aligned base)
constexpr uint32_t kStageQK = 0;          // 2 stages x 32 KB: [dk atom][q rows 0-63 | k rows 64-127][128 B]
constexpr uint32_t kStageV = 65536;       // 2 stages x 16 KB: [dv atom][64 rows][128 B]
constexpr uint32_t kHb = 98304;           // 32 KB  bf16 H^T: [dk atom][128 dv rows][128 B]
constexpr uint32_t kPt = 131072;          // 8 KB   P: [64 n rows][64 s]
constexpr uint32_t kBw = 139264;          // 8 KB   T diag(beta Gam): [n][s]
constexpr uint32_t kBu = 147456;          // 8 KB   T diag(beta): [n][s]
constexpr uint32_t kWt = 155648;          // 16 KB  W^T: [128 dk rows][64 tokens]
constexpr uint32_t kUb = 172032;          // 16 KB  U^T: [128 dv rows][64 tokens]
constexpr uint32_t kUd = 188416;          // 16 KB  U^T diag(decay)
constexpr int kLd = 68;                   // row stride (floats) of the fp32 solve matrices
constexpr uint32_t kAf = kWt;             // fp32 A [64][68] (aliases Wt/Ub/Ud during the solve)
constexpr uint32_t kTf = kWt + 64 * kLd * 4;  // fp32 T [64][68]
constexpr uint32_t kYs = kTf + 64 * kLd * 4;  // fp32 [3][16][17] solve scratch
constexpr uint32_t kVec = 204800;         // 16 x 64 floats of per-token vectors
constexpr uint32_t kBar = kVec + 16 * 256; // barriers and TMEM base
constexpr uint32_t kSmemBytes = kBar + 64 + 1024;  // + alignment slack
static_assert(kYs + 3 * 272 * 4 <= kVec, "solve scratch overlaps the vectors");

struct TcArgs {
    Problem p;
    int L;          // chunks per segment
    int fixed_segs; // segments per sequence when cu_seqlens is absent
    int auto_warm;  // 1: gate-driven warm-up for segments that do not start a sequence
    float log_eps;  // warm-up stops once the summed log decay is <= log_eps
};

__device__ __forceinline__ int nchunks_of(int64_t len) { return (int)((len + kChunk - 1) / kChunk); }

__device__ __forceinline__ uint4 pack8(const float* v) {
    uint4 w;
    w.x = pack_bf16(v[0], v[1]);
    w.y = pack_bf16(v[2], v[3]);
    w.z = pack_bf16(v[4], v[5]);
    w.w = pack_bf16(v[6], v[7]);
    return w;
}

// 32 fp32 values -> 4 swizzled 16-byte chunks (chunk0..chunk0+3) of one 128-byte row
__device__ __forceinline__ void store_row32(uint8_t* tile, int row, int chunk0, const float* v) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(tile + sw128_off(row, chunk0 + c)) = pack8(v + 8 * c);
}

// Level-D merge of the blocked inverse (D = 1, 2, 3), for the blocks (i, i-D), i = D..3:
//   Y = sum_{k=i-D}^{i-1} A_ik T_k,i-D   then   T_i,i-D = -T_ii Y.
// The diagonal blocks of T store their upper triangles as zeros, so both sums
// run over full 16-wide blocks with fixed trip counts.
template <int D>
__device__ __forceinline__ void solve_level_Y(const float* Af, const float* Tf, float* Ys, int tid) {
    constexpr int kOut = (4 - D) * 256;
#pragma unroll
    for (int q = 0; q < (kOut + kThreads - 1) / kThreads; ++q) {
        const int o = tid + q * kThreads;
        if (o < kOut) {
            const int blk = o >> 8, rr = (o >> 4) & 15, cc = o & 15;
            const int i = blk + D, j0 = i - D;
            const float* arow = Af + (16 * i + rr) * kLd + 16 * j0;
            const float* tcol = Tf + (16 * j0) * kLd + 16 * j0 + cc;
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 16 * D; ++j) s[j & 3] += arow[j] * tcol[j * kLd];
            Ys[blk * 272 + rr * 17 + cc] = (s[0] + s[1]) + (s[2] + s[3]);
        }
    }
}

template <int D>
__device__ __forceinline__ void solve_level_T(float* Tf, const float* Ys, int tid) {
    constexpr int kOut = (4 - D) * 256;
#pragma unroll
    for (int q = 0; q < (kOut + kThreads - 1) / kThreads; ++q) {
        const int o = tid + q * kThreads;
        if (o < kOut) {
            const int blk = o >> 8, rr = (o >> 4) & 15, cc = o & 15;
            const int i = blk + D, j0 = i - D;
            const float* trow = Tf + (16 * i + rr) * kLd + 16 * i;
            const float* ycol = Ys + blk * 272 + cc;
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 16; ++j) s[j & 3] += trow[j] * ycol[j * 17];
            Tf[(16 * i + rr) * kLd + 16 * j0 + cc] = -((s[0] + s[1]) + (s[2] + s[3]));
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    gdn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const TcArgs args) {
    const Problem& p = args.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* vbeta = (float*)(sm + kVec);      // beta
    float* vgam = vbeta + 64;                // gamma (natural log)
    float* vGam = vgam + 64;                 // exp(gamma)
    float* vbG = vGam + 64;                  // beta * Gam
    float* vdec = vbG + 64;                  // exp(gamma_n - gamma)
    float* va = vdec + 64;                   // row factor of E (or gamma * log2 e)
    float* vb = va + 64;                     // column factor of E
    float* vred = vb + 64;                   // reductions (8 warps)
    uint64_t* bar_tma = (uint64_t*)(sm + kBar);  // [2]
    uint64_t* bar_mma = bar_tma + 2;
    uint32_t* tmem_slot = (uint32_t*)(bar_mma + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2;                    // which half of the columns this thread takes
    const int row = ((warp & 3) << 5) | lane;    // TMEM lane (= MMA row) this thread reads
    const int Hv = p.Hv, dv = 128, dk = 128;

    // ---- which (sequence, head, segment) this CTA owns
    const int h = blockIdx.x % Hv;
    int sidx = blockIdx.x / Hv;
    int n = 0, seg = 0, segs_n = 1;
    int64_t bos = 0, len = 0;
    if (!p.cu) {
        n = sidx / args.fixed_segs;
        seg = sidx % args.fixed_segs;
        segs_n = args.fixed_segs;
        bos = (int64_t)n * p.T;
        len = p.T;
    } else {
        // warp-cooperative scan of the per-sequence segment counts (every warp
        // does the same scan, so no shared state is needed)
        int base = 0;
        bool found = false;
        for (int n0 = 0; n0 < p.N && !found; n0 += 32) {
            const int m = n0 + lane;
            int s_m = 0;
            int64_t b_m = 0, l_m = 0;
            if (m < p.N) {
                b_m = p.cu[m];
                l_m = max((int64_t)0, (int64_t)p.cu[m + 1] - b_m);
                s_m = max(1, (nchunks_of(l_m) + args.L - 1) / args.L);
            }
            int incl = s_m;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const bool mine = (m < p.N) && (sidx >= base + incl - s_m) && (sidx < base + incl);
            const unsigned bal = __ballot_sync(0xffffffffu, mine);
            if (bal) {
                const int src = __ffs(bal) - 1;
                n = __shfl_sync(0xffffffffu, m, src);
                seg = sidx - (base + __shfl_sync(0xffffffffu, incl - s_m, src));
                segs_n = __shfl_sync(0xffffffffu, s_m, src);
                bos = __shfl_sync(0xffffffffu, b_m, src);
                len = __shfl_sync(0xffffffffu, l_m, src);
                found = true;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (!found) {  // grid larger than the device offsets allow
            if (tid == 0) report(p.status, GDN_ERR_DEVICE);
            return;
        }
    }
    const int hk = h / p.group;
    const int nck = nchunks_of(len);
    const int c0 = min(nck, seg * args.L);
    const int c1 = min(nck, (seg + 1) * args.L);

    // ---- warm-up start (gate-driven); exact start from S0 when seg == 0
    int cstart = 0;
    if (seg > 0 && args.auto_warm) {
        float cum = 0.f;
        int w = c0;
        int bad = 0;
        while (w > 0 && cum > args.log_eps) {
            --w;
            const int64_t t0 = bos + (int64_t)w * kChunk;
            const int lw = (int)min((int64_t)kChunk, len - (int64_t)w * kChunk);
            // summed log decay of chunk w, and the contraction condition beta |k|^2 <= 2
            const int r = tid >> 2, q = tid & 3;
            float nrm = 0.f, gsum = 0.f;
            int viol = 0;
            if (r < lw) {
                const uint4* kr = (const uint4*)((const __nv_bfloat16*)p.k +
                                                 ((t0 + r) * p.Hk + hk) * dk + q * 32);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 u = kr[c];
                    const __nv_bfloat162* b2 = (const __nv_bfloat162*)&u;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 f = __bfloat1622float2(b2[e]);
                        nrm += f.x * f.x + f.y * f.y;
                    }
                }
            }
            nrm += __shfl_xor_sync(0xffffffffu, nrm, 1);
            nrm += __shfl_xor_sync(0xffffffffu, nrm, 2);
            if (q == 0 && r < lw) {
                const float b = p.beta[(t0 + r) * Hv + h];
                gsum = p.g[(t0 + r) * Hv + h];
                if (!(b >= 0.f && b * nrm <= 2.f)) viol = 1;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
            viol = __syncthreads_or(viol);
            if (lane == 0) vred[warp] = gsum;
            __syncthreads();
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < kThreads / 32; ++i) tot += vred[i];
            cum += tot;
            __syncthreads();
            bad |= viol;
        }
        cstart = (cum > args.log_eps || bad) ? 0 : w;
    }
    const bool exact = (cstart == 0);

    // ---- set-up: barriers, TMEM
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lane quarter
    const uint32_t sbase = smem_u32(sm);
    bool ok = true;

    // ---- initial state: H^T (lane = dv index m) from S0 or zero; this thread
    //      takes dk columns [64 wg, 64 wg + 64)
    {
        const int m = row;
        const float* s0 = (exact && p.S0) ? p.S0 + ((int64_t)n * Hv + h) * dk * dv : nullptr;
        float v[32];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int col0 = 64 * wg + 32 * hf;
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = s0 ? s0[(int64_t)(col0 + e) * dv + m] : 0.f;
            tmem_st32(tl + kColH + col0, v);
            store_row32(sm + kHb + wg * 16384, m, 4 * hf, v);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int nk = c1 - cstart;  // chunks this CTA walks (warm-up + own)
    auto issue_tma = [&](int k) {
        const int c = cstart + k;
        const int stage = k & 1;
        const int t0 = (int)(bos + (int64_t)c * kChunk);
        uint8_t* qk = sm + kStageQK + stage * 32768;
        uint8_t* vv = sm + kStageV + stage * 16384;
        mbar_arrive_expect_tx(&bar_tma[stage], 49152);
        for (int a = 0; a < 2; ++a) {
            tma_load_3d(qk + a * 16384, &tm_q, &bar_tma[stage], 64 * a, hk, t0);
            tma_load_3d(qk + a * 16384 + 8192, &tm_k, &bar_tma[stage], 64 * a, hk, t0);
            tma_load_3d(vv + a * 8192, &tm_v, &bar_tma[stage], 64 * a, h, t0);
        }
    };
    if (tid == 0 && nk > 0) issue_tma(0);

    // gates of the next chunk, loaded one chunk ahead (threads 0..63)
    float nxt_b = 0.f, nxt_g = 0.f;
    auto load_gates = [&](int k) {
        const int c = cstart + k;
        const int64_t t0 = bos + (int64_t)c * kChunk;
        const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
        nxt_b = tid < lc ? p.beta[(t0 + tid) * Hv + h] : 0.f;
        nxt_g = tid < lc ? p.g[(t0 + tid) * Hv + h] : 0.f;  // padding: g = 0
    };
    if (tid < 64 && nk > 0) load_gates(0);

    uint32_t mma_phase = 0;
    const uint32_t id_n64 = idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mn_n64 = idesc_bf16(128, 64, 1, 0);        // A MN-major
    const uint32_t id_neg_bmn_n64 = idesc_bf16(128, 64, 0, 1, 1); // -A, B MN-major
    const uint32_t id_bmn_n128 = idesc_bf16(128, 128, 0, 1);      // B MN-major, N = 128
    const float LOG2E = 1.4426950408889634f;

    for (int k = 0; k < nk && ok; ++k) {
        const int c = cstart + k;
        const int stage = k & 1;
        const bool emit = c >= c0;
        const int64_t t0 = bos + (int64_t)c * kChunk;
        const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
        const uint32_t sQK = sbase + kStageQK + stage * 32768;
        const uint32_t sV = sbase + kStageV + stage * 16384;

        // ---- MMA1 once this chunk's tiles have landed (the gates below overlap it)
        ok = __syncthreads_and(mbar_wait(&bar_tma[stage], (k >> 1) & 1));
        if (!ok) break;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + kColR1, desc_sw128(sQK + koff, 16, 1024),
                            desc_sw128(sQK + 8192 + koff, 16, 1024), id_n64, j > 0);
            }
            mma_commit(bar_mma);
            if (k + 1 < nk) issue_tma(k + 1);  // stage k+1 was freed by chunk k-1's MMAs
        }
        // ---- gates: gamma = cumsum g (per-warp scan, then warp 1 adds warp 0's total)
        if (tid < 64) {
            float x = nxt_g;
            const float b = nxt_b;
            if (k + 1 < nk) load_gates(k + 1);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            vbeta[tid] = b;
            vgam[tid] = x;
        }
        __syncthreads();
        // E_rs = exp(gamma_r - gamma_s) = a_r * b_s with a_r = exp(gamma_r - gamma_31),
        // b_s = exp(gamma_31 - gamma_s), used when every |gamma - gamma_31| < 80 (both
        // factors then stay far inside the fp32 range); else E is one exp2 per entry.
        float gr = 0.f, gm = 0.f;
        if (tid < 64) {
            const int r = tid;
            gr = vgam[r] + (r >= 32 ? vgam[31] : 0.f);
            gm = vgam[31];
            const float gl = vgam[63] + vgam[31];
            vGam[r] = expf(gr);
            vbG[r] = vbeta[r] * expf(gr);
            vdec[r] = expf(gl - gr);
        }
        const bool fac = !__syncthreads_or(tid < 64 && !(fabsf(gr - gm) < 80.f));
        if (tid < 64) {
            va[tid] = fac ? expf(gr - gm) : gr * LOG2E;
            vb[tid] = fac ? expf(gm - gr) : gr * LOG2E;
        }
        __syncthreads();

        ok = __syncthreads_and(mbar_wait(bar_mma, mma_phase));
        mma_phase ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- P (rows 0..63) and A (rows 64..127); this thread: columns [32 wg, 32 wg + 32)
        {
            float v[32];
            tmem_ld32(tl + kColR1 + 32 * wg, v);
            const int r = row & 63;
            const int s0 = 32 * wg;
            const float ar = va[r];
            if (row < 64) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = s0 + e;
                    const float E = fac ? ar * vb[s] : exp2f(ar - vb[s]);
                    v[e] = (s <= r && r < lc) ? v[e] * E : 0.f;
                }
                store_row32(sm + kPt, r, 4 * wg, v);
            } else {
                const float br = vbeta[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = s0 + e;
                    const float E = fac ? ar * vb[s] : exp2f(ar - vb[s]);
                    v[e] = (s < r && r < lc) ? br * v[e] * E : 0.f;
                }
                float4* dst = reinterpret_cast<float4*>(sm + kAf + (r * kLd + s0) * 4);
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4)
                    dst[c4] = make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^-1 in fp32: diagonal 16x16 blocks, then three merge levels
        {
            const float* Af = (const float*)(sm + kAf);
            float* Tf = (float*)(sm + kTf);
            float* Ys = (float*)(sm + kYs);
            if (tid < 64) {
                const int b = tid >> 4, cc = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s0 = (r == cc) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
                    for (int j = 0; j + 1 < r; j += 2) {
                        s0 -= Af[(16 * b + r) * kLd + 16 * b + j] * x[j];
                        s1 -= Af[(16 * b + r) * kLd + 16 * b + j + 1] * x[j + 1];
                    }
                    if (r & 1) s0 -= Af[(16 * b + r) * kLd + 16 * b + r - 1] * x[r - 1];
                    x[r] = (r < cc) ? 0.f : s0 + s1;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Tf[(16 * b + r) * kLd + 16 * b + cc] = x[r];
            }
            __syncthreads();
            solve_level_Y<1>(Af, Tf, Ys, tid);
            __syncthreads();
            solve_level_T<1>(Tf, Ys, tid);
            __syncthreads();
            solve_level_Y<2>(Af, Tf, Ys, tid);
            __syncthreads();
            solve_level_T<2>(Tf, Ys, tid);
            __syncthreads();
            solve_level_Y<3>(Af, Tf, Ys, tid);
            __syncthreads();
            solve_level_T<3>(Tf, Ys, tid);
            __syncthreads();
            // B operands of MMA_W / MMA_U: row n, columns s in [16 q, 16 q + 16), s <= n
            const int nrow = tid >> 2, q = tid & 3;
            float vw[16], vu[16];
            const float4* trow = reinterpret_cast<const float4*>(Tf + nrow * kLd + 16 * q);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 t4 = trow[c4];
                const float tt[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = 16 * q + 4 * c4 + e;
                    const float t = (s <= nrow) ? tt[e] : 0.f;
                    vw[4 * c4 + e] = t * vbG[s];
                    vu[4 * c4 + e] = t * vbeta[s];
                }
            }
            *reinterpret_cast<uint4*>(sm + kBw + sw128_off(nrow, 2 * q)) = pack8(vw);
            *reinterpret_cast<uint4*>(sm + kBw + sw128_off(nrow, 2 * q + 1)) = pack8(vw + 8);
            *reinterpret_cast<uint4*>(sm + kBu + sw128_off(nrow, 2 * q)) = pack8(vu);
            *reinterpret_cast<uint4*>(sm + kBu + sw128_off(nrow, 2 * q + 1)) = pack8(vu + 8);
        }
        fence_proxy_async();
        __syncthreads();

        // ---- MMA_W: W^T = K^T Bw^T  and  MMA_U: Ut^T = V^T Bu^T
        if (tid == 0) {
            tc_fence_after();
            if (emit) {  // MMA_HQ: H^T Q^T with the chunk-entry state (read by the epilogue)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                    mma_bf16_ss(tmem + kColHQ, desc_sw128(sbase + kHb + koff, 16, 1024),
                                desc_sw128(sQK + koff, 16, 1024), id_n64, j > 0);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mma_bf16_ss(tmem + kColR1, desc_sw128(sQK + 8192 + j * 2048, 16384, 1024),
                            desc_sw128(sbase + kBw + j * 32, 16, 1024), id_mn_n64, j > 0);
                mma_bf16_ss(tmem + kColR2, desc_sw128(sV + j * 2048, 8192, 1024),
                            desc_sw128(sbase + kBu + j * 32, 16, 1024), id_mn_n64, j > 0);
            }
            mma_commit(bar_mma);
        }
        ok = __syncthreads_and(mbar_wait(bar_mma, mma_phase));
        mma_phase ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- W^T (lane = dk index) -> bf16 rows of the MN-major B operand of MMA_HW
        {
            float v[32];
            tmem_ld32(tl + kColR1 + 32 * wg, v);
            store_row32(sm + kWt, row, 4 * wg, v);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- MMA_HW: U^T = Ut^T - H^T W^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ss(tmem + kColR2, desc_sw128(sbase + kHb + koff, 16, 1024),
                            desc_sw128(sbase + kWt + j * 2048, 8192, 1024), id_neg_bmn_n64, 1);
            }
            mma_commit(bar_mma);
        }
        ok = __syncthreads_and(mbar_wait(bar_mma, mma_phase));
        mma_phase ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- U^T (lane = dv index) -> Ub and Ud = U^T diag(decay); H^T <- Gam_n H^T
        {
            float v[32];
            tmem_ld32(tl + kColR2 + 32 * wg, v);
            if (emit) store_row32(sm + kUb, row, 4 * wg, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= vdec[32 * wg + e];
            store_row32(sm + kUd, row, 4 * wg, v);
            const float Gn = vGam[63];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t col = kColH + 64 * wg + 32 * hf;
                tmem_ld32(tl + col, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= Gn;
                tmem_st32(tl + col, v);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- MMA_UP: U^T P^T;  MMA_H: H^T += Ud K
        if (tid == 0) {
            tc_fence_after();
            if (emit) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16_ss(tmem + kColUP, desc_sw128(sbase + kUb + j * 32, 16, 1024),
                                desc_sw128(sbase + kPt + j * 32, 16, 1024), id_n64, j > 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_bf16_ss(tmem + kColH, desc_sw128(sbase + kUd + j * 32, 16, 1024),
                            desc_sw128(sQK + 8192 + j * 2048, 16384, 1024), id_bmn_n128, 1);
            mma_commit(bar_mma);
        }
        ok = __syncthreads_and(mbar_wait(bar_mma, mma_phase));
        mma_phase ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- output o[t0+n][h][m] = Gam_n (H^T Q^T)[m][n] + (U^T P^T)[m][n], n in this half
        if (emit) {
            const int m = row;
            float hq[32], up[32];
            tmem_ld32(tl + kColHQ + 32 * wg, hq);
            tmem_ld32(tl + kColUP + 32 * wg, up);
            __nv_bfloat16* op = (__nv_bfloat16*)p.o + ((t0 + 32 * wg) * Hv + h) * dv + m;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int nn = 32 * wg + e;
                if (nn < lc) op[(int64_t)e * Hv * dv] = __float2bfloat16_rn(vGam[nn] * hq[e] + up[e]);
            }
        }
        // ---- bf16 copy of the new state (dk columns [64 wg, 64 wg + 64)) for the next chunk
        {
            float v[32];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tmem_ld32(tl + kColH + 64 * wg + 32 * hf, v);
                store_row32(sm + kHb + wg * 16384, row, 4 * hf, v);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
    }

    if (!ok) {
        if (tid == 0) report(p.status, GDN_ERR_TIMEOUT);
    } else if (p.ST && seg == segs_n - 1) {
        // final state S_T = H (stored [dk][dv]): thread (m, wg) writes column m, dk half wg
        float* st = p.ST + ((int64_t)n * Hv + h) * dk * dv + row;
        float v[32];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int col0 = 64 * wg + 32 * hf;
            tmem_ld32(tl + kColH + col0, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) st[(int64_t)(col0 + e) * dv] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;  // resolved once per process (a driver entry point)
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// [T_total, H, 128] bf16 viewed as (d, head, token); box 64 x 1 x 64, 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, int64_t T_total, int H) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)std::max<int64_t>(T_total, 1)};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Segments of L chunks: count and estimated makespan in chunk-steps.
struct SplitChoice {
    int L;
    int64_t ctas;
};

SplitChoice choose_split(const std::vector<int>& nchunks, int Hv, int split_mode, int nsm) {
    int maxc = 1;
    for (int c : nchunks) maxc = std::max(maxc, c);
    auto count = [&](int L) {
        int64_t s = 0;
        for (int c : nchunks) s += std::max(1, (c + L - 1) / L);
        return s * Hv;
    };
    if (split_mode == 1) return {maxc, count(maxc)};
    if (split_mode == 2) {
        const int L = std::max(1, std::min(maxc, 2));
        return {L, count(L)};
    }
    int bestL = maxc;
    double best = 1e300;
    for (int L = 1; L <= maxc; ++L) {
        const int64_t S = count(L);
        const double waves = std::ceil((double)S / nsm);
        const double est = waves * (L + (L < maxc ? 1.5 : 0.0));
        if (est < best - 1e-9 || (std::fabs(est - best) < 1e-9 && L > bestL)) {
            best = est;
            bestL = L;
        }
    }
    return {bestL, count(bestL)};
}

std::vector<int> chunk_counts(const Problem& p, const int32_t* cu_host) {
    std::vector<int> v;
    if (!p.cu) {
        v.assign(p.N, (p.T + kChunk - 1) / kChunk);
    } else {
        v.resize(p.N);
        for (int n = 0; n < p.N; ++n) v[n] = (cu_host[n + 1] - cu_host[n] + kChunk - 1) / kChunk;
    }
    return v;
}

}  // namespace

bool tc_fwd_supported(const Problem& p) {
    return p.dtype == GDN_BF16 && p.dk == 128 && p.dv == 128;
}

size_t tc_fwd_workspace(const Problem&) { return 0; }
int tc_fwd_launches(const Problem&) { return 1; }

gdn_status launch_fwd_tc(const FwdPlan& plan, char*, cudaStream_t s) {
    const Problem& p = plan.p;
    TcArgs a;
    a.p = p;
    const std::vector<int> nck = chunk_counts(p, plan.cu_host);
    const SplitChoice sc = choose_split(nck, p.Hv, plan.split_mode, sm_count());
    a.L = sc.L;
    a.fixed_segs = p.cu ? 0 : std::max(1, (nck.empty() ? 1 : (nck[0] + sc.L - 1) / sc.L));
    a.auto_warm = plan.split_mode == 1 ? 0 : 1;
    a.log_eps = (float)(-30.0 * std::log(2.0));
    CUtensorMap mq, mk, mv;
    const int64_t Tt = std::max<int64_t>(p.T_total, 1);
    if (!make_map(&mq, p.q, Tt, p.Hk) || !make_map(&mk, p.k, Tt, p.Hk) || !make_map(&mv, p.v, Tt, p.Hv))
        return GDN_ERR_CUDA;
    if (cudaFuncSetAttribute(gdn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (sc.ctas > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    gdn_fwd_tc_kernel<<<(unsigned)sc.ctas, kThreads, kSmemBytes, s>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
