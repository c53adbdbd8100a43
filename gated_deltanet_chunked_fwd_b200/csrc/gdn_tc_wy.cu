// gdn_tc_wy.cu -- the WY / UT step of the chunked gated delta rule for bf16 tensors with
// dk = 128 on sm_100a: for every (chunk, value head), independently of the state,
//   gamma = in-chunk cumsum of g,   E_rs = exp(gamma_r - gamma_s),
//   A     = strictly-lower(diag(beta) (K K^T o E)),
//   T     = (I + A)^-1,
// written to the workspace as one bf16 64 x 64 image per (chunk, value head) in the
// 128-byte-swizzled layout that tcgen05 reads as an MMA operand (row n, 16-byte chunk c at
// chunk position c ^ (n & 7)).  The forward's state chain then forms
// W = T diag(beta Gam) K and Ut = T diag(beta) V from it.  This is the per-chunk WY / UT
// step of the chunked form of the gated delta rule (the GDN layer of the FlashQLA pages,
// news.hamidun.com "What is FlashQLA"; the pages print no formula, the chunk algebra is
// the one restated in gdn_internal.cuh).
//
// The work per chunk is small and latency-bound (a 64 x 64 x 128 Gram block and a 64 x 64
// triangular inverse), so the kernel is built for many chunks in flight rather than for one
// fast chunk: 128 threads and about 39 KB of shared memory per CTA, five CTAs per SM.  The
// Gram block K K^T is formed with warp-level mma.sync (bf16 in, fp32 out): its fragments
// stay in registers, where the gate scaling turns them into A without a TMEM round trip.
// The inverse is the blocked fp32 solve of gdn_tc_common.cuh.
#include <cuda.h>
#include <cuda_bf16.h>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kWyThreads = 128;
constexpr int kWyMinBlocks = 5;  // CTAs per SM the shared memory and registers are sized for
// shared memory (bytes from a 128-aligned base)
constexpr uint32_t wK = 0;                                 // 16 KB bf16 K [dk half][64 rows][128 B];
                                                           // then fp32 A [64][64] (as_idx layout)
constexpr uint32_t wM = 16384;                             // fp32 [64][kLd] T
constexpr uint32_t wYs = wM + 64 * kLd * 4;                // fp32 [3][16][kLdY] solve scratch
constexpr uint32_t wVec = wYs + 3 * 16 * kLdY * 4;         // beta, gamma, a, b: 4 x 64 fp32
constexpr uint32_t wSmemBytes = wVec + 4 * 64 * 4 + 128;   // + alignment slack
static_assert(wSmemBytes * kWyMinBlocks + kWyMinBlocks * 1024 <= 228 * 1024, "five CTAs per SM");

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
    gdn_wy_tc_kernel(const Problem p, uint8_t* __restrict__ timg) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, hk = h / p.group, Hv = p.Hv;
    int n = 0, c = 0;
    int64_t bos = 0, len = 0;
    if (!locate_slot(p, blockIdx.x, &n, &c, &bos, &len)) return;  // CTA-uniform
    const int64_t t0 = bos + (int64_t)c * kChunk;
    const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);

    // ---- K tile -> shared memory, 128-byte swizzled; rows past the chunk are zero
    {
        const uint4* kg = reinterpret_cast<const uint4*>(p.k);
        uint4 u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int L = i * kWyThreads + tid, r = L >> 4, ch = L & 15;
            u[i] = r < lc ? __ldg(kg + ((t0 + r) * p.Hk + hk) * 16 + ch) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int L = i * kWyThreads + tid, r = L >> 4, ch = L & 15;
            *reinterpret_cast<uint4*>(sm + wK + (ch >> 3) * 8192 + sw128_off(r, ch & 7)) = u[i];
        }
    }

    // ---- gates: gamma = cumsum g (two warp scans), E_rs = a_r b_s when factorable
    float* vbeta = (float*)(sm + wVec);
    float* vgam = vbeta + 64;
    float* va = vbeta + 128;
    float* vb = vbeta + 192;
    float gr = 0.f;
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
    const float gm = vgam[31];
    if (tid < 64) gr = vgam[tid] + (tid >= 32 ? gm : 0.f);
    // E_rs = exp(gamma_r - gamma_s) = a_r b_s, a_r = exp(gamma_r - gamma_31),
    // b_s = exp(gamma_31 - gamma_s), while every |gamma - gamma_31| < 80; else one exp2 per entry
    const bool fac = !__syncthreads_or(tid < 64 && !(fabsf(gr - gm) < 80.f));
    if (tid < 64) {
        const float LOG2E = 1.4426950408889634f;
        va[tid] = fac ? expf(gr - gm) : gr * LOG2E;
        vb[tid] = fac ? expf(gm - gr) : gr * LOG2E;
    }

    // ---- K K^T, lower block triangle: warp w owns rows 16w..16w+15, column tiles 0..2w+1
    const int g8 = lane >> 2, t4 = lane & 3;
    const int ntiles = 2 * warp + 2;
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    __syncthreads();  // K tile, vectors
    {
        const uint32_t sK = smem_u32(sm + wK);
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {  // pairs of 16-wide k steps
            const uint32_t half = sK + (kk >> 2) * 8192;
            const int ch = 2 * (kk & 3);
            uint32_t a0[4], a1[4];
            const int arow = 16 * warp + (lane & 15);
            ldsm_x4(a0, half + sw128_off(arow, ch + (lane >> 4)));
            ldsm_x4(a1, half + sw128_off(arow, ch + 2 + (lane >> 4)));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < ntiles) {  // warp-uniform
                    uint32_t b[4];
                    ldsm_x4(b, half + sw128_off(8 * j + (lane & 7), ch + (lane >> 3)));
                    mma_16816(acc[j], a0, b[0], b[1]);
                    mma_16816(acc[j], a1, b[2], b[3]);
                }
            }
        }
    }
    __syncthreads();  // every warp is done with the K tile: A overwrites it

    // ---- A = strictly-lower(beta_r (K K^T)_rs E_rs) -> shared memory (fp32)
    float* As = (float*)(sm + wK);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j < ntiles) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 16 * warp + g8 + 8 * hr, s = 8 * j + 2 * t4;
                const float ar = va[r], br = vbeta[r];
                float2 w;
                const float e0 = fac ? ar * vb[s] : exp2f(ar - vb[s]);
                const float e1 = fac ? ar * vb[s + 1] : exp2f(ar - vb[s + 1]);
                w.x = (s < r && r < lc) ? br * acc[j][2 * hr] * e0 : 0.f;
                w.y = (s + 1 < r && r < lc) ? br * acc[j][2 * hr + 1] * e1 : 0.f;
                *reinterpret_cast<float2*>(As + as_idx(r, s)) = w;
            }
        }
    }
    __syncthreads();

    // ---- T = (I + A)^-1: diagonal 16 x 16 blocks, then three merge levels
    float* M = (float*)(sm + wM);
    float* Ys = (float*)(sm + wYs);
    solve_diag(As, M, tid);
    __syncthreads();
    solve_level_Y<1, kWyThreads>(As, M, Ys, tid);
    __syncthreads();
    solve_level_T<1, kWyThreads>(M, Ys, tid);
    __syncthreads();
    solve_level_Y<2, kWyThreads>(As, M, Ys, tid);
    __syncthreads();
    solve_level_T<2, kWyThreads>(M, Ys, tid);
    __syncthreads();
    solve_level_Y<3, kWyThreads>(As, M, Ys, tid);
    __syncthreads();
    solve_level_T<3, kWyThreads>(M, Ys, tid);
    __syncthreads();

    // ---- bf16 image: thread = (row nr, half of the columns); zeros above the diagonal
    {
        const int nr = tid >> 1, hf = tid & 1;
        uint8_t* img = timg + (img_slot(bos, n, c) * Hv + h) * (int64_t)kTImgBytes;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int chunk = 4 * hf + cc, s0 = 8 * chunk;
            const float4 x0 = *reinterpret_cast<const float4*>(M + nr * kLd + s0);
            const float4 x1 = *reinterpret_cast<const float4*>(M + nr * kLd + s0 + 4);
            float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = (s0 + e <= nr) ? v[e] : 0.f;
            *reinterpret_cast<uint4*>(img + sw128_off(nr, chunk)) = pack8(v);
        }
    }
}

}  // namespace

gdn_status launch_wy_tc(const Problem& p, uint8_t* timg, cudaStream_t s) {
    if (p.num_chunks <= 0) return GDN_OK;
    const int64_t slots = img_slots(p);
    if (slots > 0x7fffffff || p.Hv > 65535) return GDN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(gdn_wy_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)wSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    const dim3 grid((unsigned)slots, (unsigned)p.Hv);
    gdn_wy_tc_kernel<<<grid, kWyThreads, wSmemBytes, s>>>(p, timg);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t wy_tc_workspace(const Problem& p) {
    return p.num_chunks > 0 ? (size_t)img_slots(p) * p.Hv * kTImgBytes : 0;
}

}  // namespace gdn
