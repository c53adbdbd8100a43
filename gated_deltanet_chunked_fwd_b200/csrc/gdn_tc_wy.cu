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
// The inverse is blocked: the four 16 x 16 diagonal blocks by fp32 substitution, then three
// merge levels on the tensor cores (warp mma.sync in tf32).
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
                                                           // then fp32 A [64][kLd]
constexpr uint32_t wM = 64 * kLd * 4;                      // fp32 [64][kLd] T
constexpr uint32_t wYs = wM + 64 * kLd * 4;                // fp32 [4 warps][16][9] merge scratch
constexpr uint32_t wVec = wYs + 3 * 16 * kLdY * 4;         // beta, gamma, a, b, |k|^2: 5 x 64 fp32
constexpr uint32_t wSmemBytes = wVec + 5 * 64 * 4 + 128;   // + alignment slack
static_assert(4 * 16 * 9 * 4 <= 3 * 16 * kLdY * 4, "merge scratch fits");
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

// fp32 -> tf32 (round to nearest, ties away), as the 32-bit pattern mma.sync reads
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D += A B for one 16 x 8 x 8 tile in tf32 (A row-major, B column-major, D fp32)
__device__ __forceinline__ void mma_tf32(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// D += A B with fp32 operands rounded to tf32.  In the merges below this adds a relative error
// of about 1e-6 (|T - T_exact| / |T| over random chunks of the workloads' distributions), some
// thirty times below the bf16 rounding that the T image gets afterwards.
__device__ __forceinline__ void mma_tf32_rn(float* d, const float* a, const float* b) {
    const uint32_t ar[4] = {to_tf32(a[0]), to_tf32(a[1]), to_tf32(a[2]), to_tf32(a[3])};
    const uint32_t br[2] = {to_tf32(b[0]), to_tf32(b[1])};
    mma_tf32(d, ar, br);
}

// The four 16 x 16 diagonal blocks of T (threads 0..63: block t / 16, column t % 16): unit
// lower-triangular inverse by forward substitution, written with zeros above the diagonal.
// A and T are [64][kLd] row-major, so every A element is read at a compile-time offset from
// the block origin.
__device__ __forceinline__ void diag_inverse(const float* As, float* M, int t) {
    if (t < 64) {
        const int b = t >> 4, cc = t & 15;
        const float* a = As + 16 * b * (kLd + 1);
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s0 = (r == cc) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j + 1 < r; j += 2) {
                s0 -= a[r * kLd + j] * x[j];
                s1 -= a[r * kLd + j + 1] * x[j + 1];
            }
            if (r & 1) s0 -= a[r * kLd + r - 1] * x[r - 1];
            x[r] = (r < cc) ? 0.f : s0 + s1;
        }
        float* m = M + 16 * b * (kLd + 1) + cc;
#pragma unroll
        for (int r = 0; r < 16; ++r) m[r * kLd] = x[r];
    }
}

// Level D (1..3) of the blocked inverse on the tensor cores: for the blocks (i, j0 = i - D),
//   Y = sum_{k = j0}^{i-1} A_ik T_k,j0,   T_i,j0 = -T_ii Y      (16 x 16 blocks)
// A work unit is one 8-column half of one block (one m16n8 tile); warp w takes units w, w + 4.
// Y goes from the accumulator layout to the B-operand layout through a per-warp 16 x 9 scratch.
template <int D>
__device__ __forceinline__ void merge_level(const float* As, float* M, float* ysw, int warp, int lane) {
    constexpr int kUnits = 2 * (4 - D);
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int u = warp; u < kUnits; u += 4) {
        const int i = D + (u >> 1), j0 = i - D, col = 16 * j0 + 8 * (u & 1);
        const int r0 = 16 * i + g, r1 = r0 + 8;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kb = 0; kb < D; ++kb) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int kc = 16 * (j0 + kb) + 8 * ks;
                const float a[4] = {As[r0 * kLd + kc + t], As[r1 * kLd + kc + t],
                                    As[r0 * kLd + kc + t + 4], As[r1 * kLd + kc + t + 4]};
                const float b[2] = {M[(kc + t) * kLd + col + g], M[(kc + t + 4) * kLd + col + g]};
                mma_tf32_rn(y, a, b);
            }
        }
        ysw[g * 9 + 2 * t] = y[0];
        ysw[g * 9 + 2 * t + 1] = y[1];
        ysw[(g + 8) * 9 + 2 * t] = y[2];
        ysw[(g + 8) * 9 + 2 * t + 1] = y[3];
        __syncwarp();
        float r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int kc = 16 * i + 8 * ks;
            const float a[4] = {M[r0 * kLd + kc + t], M[r1 * kLd + kc + t], M[r0 * kLd + kc + t + 4],
                                M[r1 * kLd + kc + t + 4]};
            const float b[2] = {ysw[(8 * ks + t) * 9 + g], ysw[(8 * ks + t + 4) * 9 + g]};
            mma_tf32_rn(r, a, b);
        }
        __syncwarp();  // the scratch is rewritten by this warp's next unit
        *reinterpret_cast<float2*>(M + r0 * kLd + col + 2 * t) = make_float2(-r[0], -r[1]);
        *reinterpret_cast<float2*>(M + r1 * kLd + col + 2 * t) = make_float2(-r[2], -r[3]);
    }
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
    gdn_wy_tc_kernel(const Problem p, uint8_t* __restrict__ timg, float2* __restrict__ summ) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
    // the forward's state-chain kernel may be scheduled as soon as every CTA of this grid has
    // started (it waits for this grid's completion before reading the images)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    float* vnrm = vbeta + 256;
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
    __syncthreads();  // K tile, vectors
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
    __syncthreads();  // every warp is done with the K tile: A overwrites it

    // ---- A = strictly-lower(beta_r (K K^T)_rs E_rs) -> shared memory (fp32); the diagonal of
    // K K^T gives |k_r|^2 for the chunk summary
    float* As = (float*)(sm + wK);
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const bool inA = i < nA;
        const int m = inA ? mA : mB, j = inA ? jA + i : jB + (i - nA);
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int r = 16 * m + g8 + 8 * hr, s = 8 * j + 2 * t4;
            const float ar = va[r], br = vbeta[r];
            const float2 b2 = *reinterpret_cast<const float2*>(vb + s);
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
            *reinterpret_cast<float2*>(As + r * kLd + s) = w;
            if (s == r) vnrm[r] = acc[i][2 * hr];
            if (s + 1 == r) vnrm[r] = acc[i][2 * hr + 1];
        }
    }
    // Chunk summary for the forward's gate-driven split: the summed log decay of the chunk and
    // whether some token breaks 0 <= beta |k|^2 <= 2 (the condition under which each token's
    // state map has norm <= exp(g)).
    const bool viol = __syncthreads_or(tid < lc && !(vbeta[tid] >= 0.f && vbeta[tid] * vnrm[tid] <= 2.f));
    if (tid == 63) summ[img_slot(bos, n, c) * Hv + h] = make_float2(gr, viol ? 1.f : 0.f);

    // ---- T = (I + A)^-1: diagonal 16 x 16 blocks, then three merge levels
    float* M = (float*)(sm + wM);
    float* Ys = (float*)(sm + wYs);
    diag_inverse(As, M, tid);
    __syncthreads();
    float* ysw = Ys + warp * 16 * 9;
    merge_level<1>(As, M, ysw, warp, lane);
    __syncthreads();
    merge_level<2>(As, M, ysw, warp, lane);
    __syncthreads();
    merge_level<3>(As, M, ysw, warp, lane);
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

gdn_status launch_wy_tc(const Problem& p, uint8_t* ws, cudaStream_t s) {
    if (p.num_chunks <= 0) return GDN_OK;
    const int64_t slots = img_slots(p);
    if (slots > 0x7fffffff || p.Hv > 65535) return GDN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(gdn_wy_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)wSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    const dim3 grid((unsigned)slots, (unsigned)p.Hv);
    gdn_wy_tc_kernel<<<grid, kWyThreads, wSmemBytes, s>>>(p, ws, (float2*)(ws + wy_tc_summary_offset(p)));
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// workspace: the T images, then one float2 summary per (image slot, value head)
size_t wy_tc_summary_offset(const Problem& p) { return (size_t)img_slots(p) * p.Hv * kTImgBytes; }
size_t wy_tc_workspace(const Problem& p) {
    return p.num_chunks > 0 ? align_up(wy_tc_summary_offset(p), 256) + (size_t)img_slots(p) * p.Hv * 8 : 0;
}

}  // namespace gdn
