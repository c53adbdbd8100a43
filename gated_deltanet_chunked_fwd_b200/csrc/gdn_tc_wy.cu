// gdn_tc_wy.cu -- the WY / UT step of the chunked gated delta rule for bf16 tensors with
// dk = 128 on sm_100a: for every (chunk, value head), independently of the state,
//   gamma = in-chunk cumsum of g,   E_rs = exp(gamma_r - gamma_s),
//   A     = strictly-lower(diag(beta) (K K^T o E)),
//   T     = (I + A)^-1,   Bw = T diag(beta Gam),   Bu = T diag(beta)   (Gam = exp(gamma)),
// written to the workspace as three bf16 64 x 64 images per (chunk, value head) in the
// 128-byte-swizzled layout that tcgen05 reads as an MMA operand (row n, 16-byte chunk c at
// chunk position c ^ (n & 7)).  The forward's state chain then forms W = Bw K and
// Ut = Bu V on the tensor cores; the backward reads all three.  This is the per-chunk WY / UT
// step of the chunked form of the gated delta rule (the GDN layer of the FlashQLA pages,
// news.hamidun.com "What is FlashQLA"; the pages print no formula, the chunk algebra is
// the one restated in gdn_internal.cuh).
//
// The work per chunk is small and latency-bound (a 64 x 64 x 128 Gram block and a 64 x 64
// triangular inverse), so the kernel is built for many chunks in flight rather than for one
// fast chunk: 128 threads, 72 registers and about 23 KB of shared memory per CTA, seven CTAs
// per SM, so that a 4096-token, 16-head call (1024 chunks) runs as one wave.  The K tile
// comes in by TMA.  The Gram block K K^T is formed with warp-level mma.sync (bf16 in, fp32
// out): its fragments stay in registers, where the gate scaling turns them into A without a
// TMEM round trip.  The inverse is blocked: the four 16 x 16 diagonal blocks by fp32
// substitution, then three merge levels on the tensor cores (warp mma.sync in tf32).
//
// A and T share one fp32 64 x 64 array X: A is strictly lower and T unit lower-triangular,
// so A sits below the diagonal and T (off its unit diagonal) above it, transposed:
// X[r][s] = A[r][s] and X[s][r] = T[r][s] for r > s.  Every X entry that feeds a merge is
// stored already rounded to tf32 (round to nearest, ties away), so the merges issue no
// conversions; the diagonal blocks of A stay fp32 for the substitution.
#include <cuda.h>
#include <cuda_bf16.h>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"
#include "gdn_tc_common.cuh"
#include "gdn_tc_inverse.cuh"

namespace gdn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kWyThreads = 128;
constexpr int kWyMinBlocks = 7;  // CTAs per SM the shared memory and registers are sized for
// shared memory (bytes from a 1024-aligned base: the TMA destination is 128-byte swizzled)
constexpr uint32_t wK = 0;                          // 16 KB bf16 K [dk half][64 rows][128 B];
                                                    // then fp32 X [64][kXs]
constexpr uint32_t wYs = 64 * kXs * 4;              // fp32 [4 warps][16][9] merge scratch
constexpr uint32_t wVec = wYs + 4 * 16 * 9 * 4;     // beta, gamma, a, b, |k|^2, beta Gam: 6 x 64 fp32
constexpr uint32_t wBar = wVec + 6 * 64 * 4;        // mbarrier of the K tile
constexpr uint32_t wSmemBytes = wBar + 16 + 1024;   // + alignment slack
static_assert(wYs >= 16384, "X covers the K tile it replaces");
static_assert(wSmemBytes * kWyMinBlocks + kWyMinBlocks * 1024 <= 228 * 1024, "CTAs per SM");

// 4 8x8 b16 matrices from shared memory (lane groups of 8 give the row addresses of matrix 0..3)
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D += A B for one 16 x 8 x 16 tile: A row-major bf16, B column-major bf16, D fp32
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Image slot x -> (sequence n, chunk c of it, its first token and length); false when the
// slot belongs to no chunk.  The slot of sequence n's first chunk, floor(bos_n / 64) + n, is
// strictly increasing in n, so n is found by bisection over the sequence offsets.
__device__ __forceinline__ bool locate_slot(const Problem& p, int64_t x, int* n_out, int* c_out,
                                            int64_t* bos_out, int64_t* len_out) {
    if (p.N <= 0) return false;
    auto bos_of = [&](int n) -> int64_t { return p.cu ? (int64_t)p.cu[n] : (int64_t)n * p.T; };
    int lo = 0, hi = p.N - 1;
    if (img_slot(bos_of(0), 0, 0) > x) return false;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (img_slot(bos_of(mid), mid, 0) <= x) lo = mid;
        else hi = mid - 1;
    }
    const int64_t bos = bos_of(lo);
    const int64_t len = p.cu ? max((int64_t)0, (int64_t)p.cu[lo + 1] - bos) : (int64_t)p.T;
    const int64_t c = x - img_slot(bos, lo, 0);
    if (c >= nchunks_of(len)) return false;
    *n_out = lo;
    *c_out = (int)c;
    *bos_out = bos;
    *len_out = len;
    return true;
}

__global__ void __launch_bounds__(kWyThreads, kWyMinBlocks)
    gdn_wy_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const Problem p, uint8_t* __restrict__ timg,
                     float2* __restrict__ summ) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // the forward's state-chain kernel may be scheduled as soon as every CTA of this grid has
    // started (it waits for this grid's completion before reading the images)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) prefetch_tensormap(&tm_k);  // its first use is a few hundred cycles away
    const int h = blockIdx.y, hk = h / p.group, Hv = p.Hv;
    int n = 0, c = 0;
    int64_t bos = 0, len = 0;
    if (!locate_slot(p, blockIdx.x, &n, &c, &bos, &len)) return;  // CTA-uniform
    const int64_t t0 = bos + (int64_t)c * kChunk;
    const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
    uint64_t* bar = (uint64_t*)(sm + wBar);

    // ---- K tile by TMA ([dk half][64 rows][128 B], 128-byte swizzled).  Rows past the chunk
    // (the next sequence's tokens, or zeros past the tensor's end) only reach entries of A that
    // the mask below sets to zero.  The chunk's gates are loaded meanwhile.
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    float x = 0.f, bt = 0.f;
    if (tid < lc) {  // lc <= 64
        x = p.g[(t0 + tid) * Hv + h];
        bt = p.beta[(t0 + tid) * Hv + h];
    }
    __syncthreads();  // the barrier is initialised
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, 16384);
        tma_load_3d(sm + wK, &tm_k, bar, 0, hk, (int)t0);
        tma_load_3d(sm + wK + 8192, &tm_k, bar, 64, hk, (int)t0);
    }

    // ---- gates: gamma = cumsum g (two warp scans), E_rs = a_r b_s when factorable
    float* vbeta = (float*)(sm + wVec);
    float* vgam = vbeta + 64;
    float* va = vbeta + 128;
    float* vb = vbeta + 192;
    float* vnrm = vbeta + 256;
    float* vbG = vbeta + 320;
    float gr = 0.f;
    if (tid < 64) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        vbeta[tid] = bt;
        vgam[tid] = x;
    }
    __syncthreads();
    const float gm = vgam[31];
    if (tid < 64) gr = vgam[tid] + (tid >= 32 ? gm : 0.f);
    // E_rs = exp(gamma_r - gamma_s) = a_r b_s, a_r = exp(gamma_r - gamma_31),
    // b_s = exp(gamma_31 - gamma_s), while every |gamma - gamma_31| < 80; else one exp2 per entry
    const bool fac = !__syncthreads_or(tid < 64 && !(fabsf(gr - gm) < 80.f));
    if (tid < 64) {
        const float LOG2E = 1.4426950408889634f;
        va[tid] = fac ? expf(gr - gm) : gr * LOG2E;
        vb[tid] = fac ? expf(gm - gr) : gr * LOG2E;
        vbG[tid] = bt * expf(gr);
    }

    // ---- K K^T, lower block triangle: 20 tiles of 16 rows (m-tile) x 8 columns (n-tile), five
    // per warp.  m-tiles 0 and 3 (2 + 8 tiles) are shared by warps 0 and 1, m-tiles 1 and 2
    // (4 + 6 tiles) by warps 2 and 3; a warp's tiles are one run of n-tiles in m-tile mA and
    // possibly a second run in m-tile mB.
    const int g8 = lane >> 2, t4 = lane & 3;
    int mA, jA, nA, mB, jB;
    switch (warp) {
        case 0: mA = 0; jA = 0; nA = 2; mB = 3; jB = 0; break;   // (0: 0-1), (3: 0-2)
        case 1: mA = 3; jA = 3; nA = 5; mB = 3; jB = 8; break;   // (3: 3-7)
        case 2: mA = 1; jA = 0; nA = 4; mB = 2; jB = 0; break;   // (1: 0-3), (2: 0)
        default: mA = 2; jA = 1; nA = 5; mB = 2; jB = 6; break;  // (2: 1-5)
    }
    const bool twoA = nA < 5;  // warp-uniform: a second m-tile run exists
    float acc[5][4];
#pragma unroll
    for (int i = 0; i < 5; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    __syncthreads();  // vectors
    if (!__syncthreads_and(mbar_wait(bar, 0))) {  // the K tile has landed (bounded wait)
        if (tid == 0) report(p.status, GDN_ERR_TIMEOUT);
        return;
    }
    {
        const uint32_t sK = smem_u32(sm + wK);
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {  // pairs of 16-wide k steps
            const uint32_t half = sK + (kk >> 2) * 8192;
            const int ch = 2 * (kk & 3);
            uint32_t aA0[4], aA1[4], aB0[4], aB1[4];
            ldsm_x4(aA0, half + sw128_off(16 * mA + (lane & 15), ch + (lane >> 4)));
            ldsm_x4(aA1, half + sw128_off(16 * mA + (lane & 15), ch + 2 + (lane >> 4)));
            if (twoA) {
                ldsm_x4(aB0, half + sw128_off(16 * mB + (lane & 15), ch + (lane >> 4)));
                ldsm_x4(aB1, half + sw128_off(16 * mB + (lane & 15), ch + 2 + (lane >> 4)));
            }
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                const bool inA = i < nA;  // warp-uniform
                const int j = inA ? jA + i : jB + (i - nA);
                uint32_t b[4];
                ldsm_x4(b, half + sw128_off(8 * j + (lane & 7), ch + (lane >> 3)));
                if (inA) {
                    mma_16816(acc[i], aA0, b[0], b[1]);
                    mma_16816(acc[i], aA1, b[2], b[3]);
                } else {
                    mma_16816(acc[i], aB0, b[0], b[1]);
                    mma_16816(acc[i], aB1, b[2], b[3]);
                }
            }
        }
    }
    __syncthreads();  // every warp is done with the K tile: X overwrites it

    // ---- A = strictly-lower(beta_r (K K^T)_rs E_rs) -> X (entries on and above the diagonal
    // that a tile covers are written as zeros and later overwritten by T).  Blocks below the
    // diagonal block are merge operands only: stored rounded to tf32.  The diagonal of K K^T
    // gives |k_r|^2 for the chunk summary.
    float* X = (float*)(sm + wK);
    {
        float arA[2], brA[2], arB[2], brB[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            arA[hr] = va[16 * mA + g8 + 8 * hr];
            brA[hr] = vbeta[16 * mA + g8 + 8 * hr];
            arB[hr] = va[16 * mB + g8 + 8 * hr];
            brB[hr] = vbeta[16 * mB + g8 + 8 * hr];
        }
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const bool inA = i < nA;
            const int m = inA ? mA : mB, j = inA ? jA + i : jB + (i - nA);
            const int s = 8 * j + 2 * t4;
            const bool below = (j >> 1) < m;  // warp-uniform
            const float2 b2 = *reinterpret_cast<const float2*>(vb + s);
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 16 * m + g8 + 8 * hr;
                const float ar = inA ? arA[hr] : arB[hr], br = inA ? brA[hr] : brB[hr];
                float e0, e1;
                if (fac) {  // block-uniform
                    e0 = ar * b2.x;
                    e1 = ar * b2.y;
                } else {
                    e0 = exp2f(ar - b2.x);
                    e1 = exp2f(ar - b2.y);
                }
                float2 w;
                w.x = (s < r && r < lc) ? br * acc[i][2 * hr] * e0 : 0.f;
                w.y = (s + 1 < r && r < lc) ? br * acc[i][2 * hr + 1] * e1 : 0.f;
                if (below) {
                    w.x = tf32r(w.x);
                    w.y = tf32r(w.y);
                }
                *reinterpret_cast<float2*>(X + r * kXs + s) = w;
                if (s == r) vnrm[r] = acc[i][2 * hr];
                if (s + 1 == r) vnrm[r] = acc[i][2 * hr + 1];
            }
        }
    }
    // Chunk summary for the forward's gate-driven split: the summed log decay of the chunk and
    // whether some token breaks 0 <= beta |k|^2 <= 2 (the condition under which each token's
    // state map has norm <= exp(g)).
    const bool viol = __syncthreads_or(tid < lc && !(vbeta[tid] >= 0.f && vbeta[tid] * vnrm[tid] <= 2.f));
    if (tid == 63) summ[img_slot(bos, n, c) * Hv + h] = make_float2(gr, viol ? 1.f : 0.f);

    // ---- T = (I + A)^-1: diagonal 16 x 16 blocks, then three merge levels
    {
        float xs[16];
        if (tid < 64) diag_solve(X, tid, xs);
        __syncthreads();  // every diagonal A block has been read
        if (tid < 64) diag_store(X, tid, xs);
    }
    __syncthreads();
    float* ysw = (float*)(sm + wYs) + warp * 16 * 9;
    merge_level<1>(X, ysw, warp, lane);
    __syncthreads();
    merge_level<2>(X, ysw, warp, lane);
    __syncthreads();
    merge_level<3>(X, ysw, warp, lane);
    __syncthreads();

    // ---- bf16 images T, Bw, Bu: thread = rows nr4 .. nr4 + 3, columns s0 .. s0 + 7 (one 16-byte
    // chunk of each row), from T[r][s] = X[s][r] for r > s
    {
        const int nr4 = 4 * (tid & 15), ch = tid >> 4, s0 = 8 * ch;
        uint8_t* img = timg + (img_slot(bos, n, c) * Hv + h) * (int64_t)kWyImgBytes;
        float v[4][8];
        if (s0 > nr4 + 3) {  // the block lies above the diagonal
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) v[q][e] = 0.f;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 col = *reinterpret_cast<const float4*>(X + (s0 + e) * kXs + nr4);
                v[0][e] = t_sel(col.x, nr4, s0 + e);
                v[1][e] = t_sel(col.y, nr4 + 1, s0 + e);
                v[2][e] = t_sel(col.z, nr4 + 2, s0 + e);
                v[3][e] = t_sel(col.w, nr4 + 3, s0 + e);
            }
        }
        float sw[8], su[8];
#pragma unroll
        for (int e4 = 0; e4 < 2; ++e4) {
            const float4 w4 = *reinterpret_cast<const float4*>(vbG + s0 + 4 * e4);
            const float4 u4 = *reinterpret_cast<const float4*>(vbeta + s0 + 4 * e4);
            sw[4 * e4] = w4.x; sw[4 * e4 + 1] = w4.y; sw[4 * e4 + 2] = w4.z; sw[4 * e4 + 3] = w4.w;
            su[4 * e4] = u4.x; su[4 * e4 + 1] = u4.y; su[4 * e4 + 2] = u4.z; su[4 * e4 + 3] = u4.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t off = sw128_off(nr4 + q, ch);
            float bw[8], bu[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                bw[e] = v[q][e] * sw[e];
                bu[e] = v[q][e] * su[e];
            }
            *reinterpret_cast<uint4*>(img + off) = pack8(v[q]);
            *reinterpret_cast<uint4*>(img + kTImgBytes + off) = pack8(bw);
            *reinterpret_cast<uint4*>(img + 2 * kTImgBytes + off) = pack8(bu);
        }
    }
}

}  // namespace

gdn_status tc::launch_wy_tc(const Problem& p, const CUtensorMap& tm_k, uint8_t* ws, cudaStream_t s) {
    if (p.num_chunks <= 0) return GDN_OK;
    const int64_t slots = img_slots(p);
    if (slots > 0x7fffffff || p.Hv > 65535) return GDN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(gdn_wy_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)wSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    const dim3 grid((unsigned)slots, (unsigned)p.Hv);
    gdn_wy_tc_kernel<<<grid, kWyThreads, wSmemBytes, s>>>(tm_k, p, ws,
                                                          (float2*)(ws + wy_tc_summary_offset(p)));
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// workspace: the T / Bw / Bu images, then one float2 summary per (image slot, value head)
size_t wy_tc_summary_offset(const Problem& p) { return (size_t)img_slots(p) * p.Hv * kWyImgBytes; }
size_t wy_tc_workspace(const Problem& p) {
    return p.num_chunks > 0 ? align_up(wy_tc_summary_offset(p), 256) + (size_t)img_slots(p) * p.Hv * 8 : 0;
}

}  // namespace gdn
