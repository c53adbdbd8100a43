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
// fast chunk: 128 threads, 64 registers, about 25 KB of shared memory and 64 TMEM columns per
// CTA, eight CTAs per SM, so that a 4096-token, 16-head call (1024 chunks) runs as one wave.  The
// K tile comes in by TMA.  The Gram block K K^T is one tcgen05 MMA group (M = 128, N = 64, bf16
// in, fp32 out in TMEM); two warps read its rows and scale them into A.  The inverse is blocked:
// the four 16 x 16 diagonal blocks by fp32 substitution, then three merge levels as warp-level
// tf32 MMAs (gdn_tc_inverse.cuh).
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
constexpr int kWyMinBlocks = 8;  // CTAs per SM the shared memory and registers are sized for (64 registers)
constexpr int kWyMinBlocksGrouped = 6;  // with grouped value heads: the loop over the group keeps
                                        // a few more values live (80 registers)
// shared memory (bytes from a 1024-aligned base: the TMA destination is 128-byte swizzled)
constexpr uint32_t wK = 0;                          // 16 KB bf16 K [dk half][64 rows][128 B];
                                                    // then fp32 X [64][kXs]
constexpr uint32_t wYs = 64 * kXs * 4;              // fp32 [4 warps][16][9] merge scratch
constexpr uint32_t wVec = wYs + 4 * 16 * 9 * 4;     // beta, gamma, a, b, |k|^2, beta Gam: 6 x 64 fp32
constexpr uint32_t wBar = wVec + 6 * 64 * 4;        // mbarriers of the K tile and the Gram MMA,
                                                    // TMEM base
// The Gram MMA reads its A operand as 128 rows (1024-byte groups of 8): the K tile's rows are
// 0-63; rows 64-127 of the second k-half lie 8 KB past the tile and only feed D rows 64-127,
// which are never read.  They must still lie inside this CTA's shared memory.
constexpr uint32_t wAReach = wK + 3 * 8192;
constexpr uint32_t wSmemBytes = (wBar + 32 > wAReach ? wBar + 32 : wAReach) + 1024;  // + alignment slack
constexpr uint32_t kWyTmemCols = 64;                // D = [K;*] K^T: 128 lanes x 64 fp32 columns
static_assert(wYs >= 16384, "X covers the K tile it replaces");
static_assert(wSmemBytes * kWyMinBlocks + kWyMinBlocks * 1024 <= 228 * 1024, "CTAs per SM");
static_assert(kWyTmemCols * kWyMinBlocks <= 512, "TMEM columns per SM");

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

// kGrouped: value heads share q/k heads (p.group > 1); the CTA loops over the group.  Without
// grouping the loop has one pass and compiles away.  kPrep: the input preprocessing flags
// (GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM) are compiled in.
template <bool kGrouped, bool kPrep>
__global__ void __launch_bounds__(kWyThreads, kGrouped ? kWyMinBlocksGrouped : kWyMinBlocks)
    gdn_wy_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const Problem p, uint8_t* __restrict__ timg,
                     float2* __restrict__ summ, int32_t* __restrict__ flags, int nflags,
                     int32_t* __restrict__ flags2, int nflags2, int with_t) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) prefetch_tensormap(&tm_k);  // its first use is a few hundred cycles away
    // one CTA per (chunk slot, q/k head): the Gram block of the head's K is formed once and serves
    // every value head of its group (value heads hk G .. hk G + G - 1 share k)
    const int hk = blockIdx.y, G = kGrouped ? p.group : 1, Hv = p.Hv;
    int n = 0, c = 0;
    int64_t bos = 0, len = 0;
    // the scan flags of the state chain and of the backward's reverse walks start at zero (CTA
    // (x, hk) clears entry x Hv + hk G + i of each; both have fewer CTAs than the image slots times
    // the value heads)
    if (tid < G) {
        const int64_t fi = (int64_t)blockIdx.x * Hv + hk * G + tid;
        if (fi < nflags) flags[fi] = 0;
        if (fi < nflags2) flags2[fi] = 0;
    }
    const bool live = locate_slot(p, blockIdx.x, &n, &c, &bos, &len);  // CTA-uniform
    uint64_t* bar = (uint64_t*)(sm + wBar);
    uint64_t* bar_mma = bar + 1;
    uint32_t* tmem_slot = (uint32_t*)(bar + 2);
    // TMEM for the Gram block, taken before the dependent grid may launch: that grid's CTAs take
    // all 512 columns of an SM and then wait for this grid, so they must find ours already held
    if (live && warp == 0) {
        tmem_alloc(tmem_slot, kWyTmemCols);
        tmem_relinquish();
    }
    // the forward's state-chain kernel may be scheduled as soon as every CTA of this grid has
    // started (it waits for this grid's completion before reading the images)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!live) return;
    const int64_t t0 = bos + (int64_t)c * kChunk;
    const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);

    // ---- K tile by TMA ([dk half][64 rows][128 B], 128-byte swizzled).  Rows past the chunk
    // (the next sequence's tokens, or zeros past the tensor's end) only reach entries of A that
    // the mask below sets to zero.  The first value head's gates are loaded meanwhile.
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
    }
    float xg = 0.f, bt = 0.f;
    const int glog = kPrep ? p.gate_logits : 0;  // GDN_FLAG_GATE_LOGITS, when compiled in
    auto load_gates = [&](int h) {
        // padding: g = beta = 0 (as raw gates: -inf, which the maps take to 0); raw gates are mapped
        // where they are used
        const float pad = glog ? -INFINITY : 0.f;
        xg = tid < lc ? p.g[(t0 + tid) * Hv + h] : pad;  // lc <= 64
        bt = tid < lc ? p.beta[(t0 + tid) * Hv + h] : pad;
    };
    load_gates(hk * G);
    tc_fence_before();
    __syncthreads();  // the barriers are initialised, the TMEM base is written
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, 16384);
        tma_load_3d(sm + wK, &tm_k, bar, 0, hk, (int)t0);
        tma_load_3d(sm + wK + 8192, &tm_k, bar, 64, hk, (int)t0);
    }
    float* vbeta = (float*)(sm + wVec);
    float* vgam = vbeta + 64;
    float* va = vbeta + 128;
    float* vb = vbeta + 192;
    float* vnrm = vbeta + 256;
    float* vbG = vbeta + 320;
    float* X = (float*)(sm + wK);

    // ---- K K^T on the tensor core: D = A K^T with A the K tile read as 128 rows (D rows 0-63 are
    // the Gram block; rows 64-127 come from the bytes after the tile and are not read), N = 64,
    // bf16 in, fp32 out in TMEM lanes 0-63 (one K row per lane)
    bool ok = __syncthreads_and(mbar_wait(bar, 0));  // the K tile has landed
    if (kPrep && p.qk_norm) {  // raw k rows: normalised in place before the Gram (thread pair per row)
        l2norm_row_sw128(sm + wK, 8192, tid >> 1, tid & 1);
        fence_proxy_async();
        __syncthreads();
    }
    if (ok && tid == 0) {
        const uint64_t dK = desc_sw128(smem_u32(sm + wK), 16, 1024);
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 8; ++j)  // K steps of 16: four per 64-wide k half (8 KB apart)
            mma_bf16_ss(tmem, dK + (((j >> 2) * 8192 + (j & 3) * 32) >> 4),
                        dK + (((j >> 2) * 8192 + (j & 3) * 32) >> 4), idesc_bf16(128, 64, 0, 0), j > 0);
        mma_commit(bar_mma);
    }
    if (!ok && tid == 0) report(p.status, GDN_ERR_TIMEOUT);

    for (int gi = 0; gi < G && ok; ++gi) {
    const int h = hk * G + gi;  // the value head of this pass
    // ---- gates: gamma = cumsum g (two warp scans), E_rs = a_r b_s when factorable
    float gr = 0.f;
    const float btm = gate_beta(bt, glog);  // the mapped beta of this thread's token
    if (tid < 64) {
        float x = gate_g(xg, glog);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        vbeta[tid] = btm;
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
        vbG[tid] = btm * expf(gr);
    }
    if (gi + 1 < G) load_gates(h + 1);  // the next value head's gates, while this one runs
    // the Gram block is in TMEM (the first pass waits for it) and the vectors are written
    if (gi == 0) {
        ok = __syncthreads_and(mbar_wait(bar_mma, 0));
        if (!ok) {
            if (tid == 0) report(p.status, GDN_ERR_TIMEOUT);
            break;
        }
    } else {
        __syncthreads();
    }
    {
        tc_fence_after();
        // ---- A = strictly-lower(beta_r (K K^T)_rs E_rs) -> X, row r by thread r (warps 0 and 1 read
        // TMEM lanes 0-63).  X overwrites the K tile, which the MMA has read.  Entries below the
        // diagonal 16 x 16 blocks are merge operands only: stored rounded to tf32.  The diagonal of
        // K K^T gives |k_r|^2 for the chunk summary.  Blocks above the diagonal ones are neither
        // read nor stored: their places in X receive T before anything reads them.  Warp 0 (rows
        // 0-31) has no entries in column blocks 2 and 3.
        float* X = (float*)(sm + wK);
        if (warp < 2) {
            const int r = tid;
            const float br = r < lc ? vbeta[r] : 0.f;  // rows past the chunk's end are zero
            const float ar = va[r], bra = br * ar;  // beta_r a_r
            float* xr = X + r * kXs;
            const int qn = warp == 0 ? 2 : 4;  // warp-uniform: the TMEM load is warp-collective
#pragma unroll 1
            for (int q = 0; q < qn; ++q) {  // 16 columns s = 16 q .. 16 q + 15 at a time
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + 16 * q, v);
                if ((r >> 4) == q) {  // the diagonal entry, by an unrolled select (no indexed registers)
                    float dg = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) dg = (e == (r & 15)) ? v[e] : dg;
                    vnrm[r] = dg;
                }
                // beta_r E_rs with E_rs = a_r b_s, or exp2(a_r - b_s) when the chunk's decay range
                // is too wide (block-uniform branch: one loop per form); E is used only under the
                // mask: above the diagonal it may overflow.  Entries below the diagonal 16 x 16 blocks
                // (q < r / 16) are merge operands only: stored rounded to tf32.
                const bool below = q < (r >> 4);
                const bool store = q <= (r >> 4);
                if (fac) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= bra * vb[16 * q + e];
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= br * exp2f(ar - vb[16 * q + e]);
                }
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    float o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = 16 * q + 4 * e4 + e;
                        const float x = s < r ? v[4 * e4 + e] : 0.f;
                        o[e] = below ? tf32r(x) : x;
                    }
                    if (store) *reinterpret_cast<float4*>(xr + 16 * q + 4 * e4) = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
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

    // ---- bf16 images T (for the backward only), Bw, Bu: thread = rows nr4 .. nr4 + 3, columns
    // s0 .. s0 + 7 (one 16-byte chunk of each row, all in one 16 x 16 block of T), from
    // T[r][s] = X[s][r].  X holds T^T in every block on or above its diagonal (the diagonal
    // blocks exactly, with their ones and zeros); blocks of T above the diagonal are zero.
    {
        const int nr4 = 4 * (tid & 15), ch = tid >> 4, s0 = 8 * ch;
        uint8_t* img = timg + (img_slot(bos, n, c) * Hv + h) * (int64_t)kWyImgBytes;
        float v[4][8];
        if ((s0 >> 4) > (nr4 >> 4)) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) v[q][e] = 0.f;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 col = *reinterpret_cast<const float4*>(X + (s0 + e) * kXs + nr4);
                v[0][e] = col.x;
                v[1][e] = col.y;
                v[2][e] = col.z;
                v[3][e] = col.w;
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
            if (with_t) *reinterpret_cast<uint4*>(img + off) = pack8(v[q]);  // the backward reads T
            *reinterpret_cast<uint4*>(img + kTImgBytes + off) = pack8(bw);
            *reinterpret_cast<uint4*>(img + 2 * kTImgBytes + off) = pack8(bu);
        }
    }
    __syncthreads();  // the images have read X and the vectors: the next value head may overwrite them
    }  // value heads
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kWyTmemCols);
    }
}

}  // namespace

gdn_status tc::launch_wy_tc(const Problem& p, const CUtensorMap& tm_k, uint8_t* ws, int32_t* flags, int nflags,
                            int32_t* flags2, int nflags2, bool with_t, cudaStream_t s) {
    if (p.num_chunks <= 0) return GDN_OK;
    const int64_t slots = img_slots(p);
    if (slots > 0x7fffffff || p.Hv > 65535) return GDN_ERR_UNSUPPORTED;
    const bool prep = p.gate_logits || p.qk_norm;
    auto kern = p.group > 1 ? (prep ? gdn_wy_tc_kernel<true, true> : gdn_wy_tc_kernel<true, false>)
                            : (prep ? gdn_wy_tc_kernel<false, true> : gdn_wy_tc_kernel<false, false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    const dim3 grid((unsigned)slots, (unsigned)p.Hk);
    if ((int64_t)nflags > slots * p.Hv || (int64_t)nflags2 > slots * p.Hv)
        return GDN_ERR_DEVICE;  // every flag has a CTA to clear it
    kern<<<grid, kWyThreads, wSmemBytes, s>>>(tm_k, p, ws, (float2*)(ws + wy_tc_summary_offset(p)), flags, nflags,
                                              flags2, nflags2, with_t ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// workspace: the T / Bw / Bu images, then one float2 summary per (image slot, value head)
size_t wy_tc_summary_offset(const Problem& p) { return (size_t)img_slots(p) * p.Hv * kWyImgBytes; }
size_t wy_tc_workspace(const Problem& p) {
    return p.num_chunks > 0 ? align_up(wy_tc_summary_offset(p), 256) + (size_t)img_slots(p) * p.Hv * 8 : 0;
}

}  // namespace gdn
