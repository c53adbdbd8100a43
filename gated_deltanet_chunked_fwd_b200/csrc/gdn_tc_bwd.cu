// gdn_tc_bwd.cu -- tensor-core backward of the chunked gated delta rule (bf16, dk = dv = 128,
// sm_100a).  The backward of the GDN layer (FlashQLA pages: dothoosh.com article, opening
// paragraph, "backward pass"; news.hamidun.com page, "large-scale pretraining" scenario).
//
// Three to five launches: the WY kernel (T, T diag(beta Gam), T diag(beta) images and per-chunk
// gate summaries), the fused forward kernel in replay mode (the bf16 entry state H^T of every
// chunk, as a ready-to-use 128-byte-swizzled shared-memory image), in sequences of at least four
// segments the adjoint scan's pre-pass (this kernel with kPre), this reverse kernel, and with
// grouped value heads (or GDN_FLAG_QK_L2NORM) the reduction of dq / dk over each group (and the
// chain rule of the q / k normalisation).  The reverse kernel runs one CTA per (sequence, value head, segment of
// chunks), 256 threads: the two warps of each TMEM lane quarter share its lanes (thread <-> MMA
// row) and split each row's columns, or tokens, in halves.  A segment walks its chunks
// backwards with the state adjoint dH (fp32, TMEM).  Its exit adjoint comes from a reverse
// warm-up: the adjoint map of a chunk, dH -> (Gam_n I - W^T Kd) dH, is the transpose of the
// chunk's state map and has the same norm bound exp(sum g) while 0 <= beta |k|^2 <= 2, so a
// segment that does not end its sequence starts from dH = 0 a few chunks later (until the summed
// log decay reaches log eps) and runs only the dH chain there.  Where that warm-up fails, or
// would be long, the segment starts exactly from the entry adjoint that the adjoint scan's
// pre-pass recorded (in sequences of at least four segments), else from dS_T at the sequence
// end.  Every chunk maps the adjoint affinely, dH_c = (Gam_n I - W^T Kd) dH_c+1 + b_c, so the
// scan is the forward's affine scan run backwards over the segments.  Per chunk (notation of
// gdn_internal.cuh; E, Gam, dec, beta from the gates; Kb = diag(beta Gam) K):
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
#include <type_traits>
#include <vector>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kNT = 256;
constexpr int kTmemColsB = 512;
// TMEM columns (lane = MMA row)
constexpr uint32_t cH = 0;     // dH^T fp32                                      [0, 128)
constexpr uint32_t cHb = 128;  // bf16 dH^T (A operand)                          [128, 192)
constexpr uint32_t cR1 = 192;  // Q K^T / K K^T, later dk^T (main part)
constexpr uint32_t cR2 = 256;  // W^T, later TdU^T, later dKd^T
constexpr uint32_t cR3 = 320;  // Ut^T -> U^T, later [dP ; dA'], later K^T (dP o E)^T
constexpr uint32_t cR4 = 384;  // dO^T P, later H dO^T
constexpr uint32_t cR5 = 448;  // dH^T K^T, then bf16 dU^T (cols 0..31), later H TdU^T = -TdW^T
                               // (the second half of one N = 128 product with R4)

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t bQK = 0;        // 32 KB [dk atom][q rows 0-63 | k rows 64-127][128 B]
constexpr uint32_t bV = 32768;     // 16 KB [dv atom][64 rows][128 B]; phase 2: fp32 G [64][64]
constexpr uint32_t bDO = 49152;    // 32 KB [dv atom][do rows 0-63 | TdU rows 64-127][128 B]
constexpr uint32_t bHt = 81920;    // 32 KB bf16 H^T [dk atom][128 dv rows][128 B]
constexpr uint32_t bT = 114688;    // 8 KB  T [64 rows s][64 r]; later S = G + G^T [s][j]
constexpr uint32_t bBw = 122880;   // 8 KB  T diag(beta Gam); later diag(Gam) Q [atom][64][128]
constexpr uint32_t bBu = 131072;   // 8 KB  T diag(beta)      (over Bw + Bu)
// T, Bw, Bu arrive together: one copy of the WY step's three images
static_assert(bBw == bT + kTImgBytes && bBu == bBw + kTImgBytes, "WY images are contiguous");
constexpr uint32_t bP = 139264;    // 8 KB  P [64 r][64 s]; later dP o E
constexpr uint32_t bWt = 147456;   // 16 KB -W^T [128 dk rows][64 s]
constexpr uint32_t bUt = 163840;   // 16 KB U^T [128 dv rows][64 s]
constexpr uint32_t bDHt = 180224;  // 32 KB bf16 dH^T [dk atom][128 dv rows][128 B]
constexpr uint32_t bVec = 212992;  // per-token vectors (8 x 64 floats)
constexpr uint32_t bRed = bVec + 2048;  // reductions [4][64] floats + accumulators [4][64]
constexpr uint32_t bBar = bRed + 2048;
constexpr uint32_t kSmemB = bBar + 64 + 1024;

constexpr uint32_t kHImg = 32768;  // bytes of one saved H^T image
constexpr int kRevScanMinSegs = 4;  // the adjoint scan is used in sequences of at least four segments
constexpr int kRevScanFoldAllowance = 16;  // fold products, in dH-chain chunk steps

struct TcBwdArgs {
    BwdProblem b;
    const uint8_t* himg;  // H^T entry-state images, by (image slot, value head)
    const uint8_t* timg;  // T / Bw / Bu images of the WY step, by (image slot, value head)
    const float2* summ;   // per (image slot, value head): summed log decay, norm-condition flag
    float* dqw;           // [T_total][Hv][dk] per-value-head dq
    float* dkw;           // [T_total][Hv][dk] per-value-head dk
    int L;                // chunks per segment
    int fixed_segs;       // segments per sequence when cu_seqlens is absent
    int auto_warm;        // 1: reverse warm-up for segments that do not end their sequence
    // adjoint affine scan for segments whose reverse warm-up cannot reach log_eps: per CTA a flag
    // and three fp32 [dk][dv] records (exit adjoint, M, B); nullptr (no sequence has enough
    // segments): such a segment replays the dH chain from dS_T at the sequence end instead
    int32_t* scan_flags;
    float* scan_rec;
    float log_eps;        // the warm-up stops once the summed log decay is <= log_eps
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

// End (exclusive) of the reverse warm-up of the segment whose chunks end at c1: the smallest w > c1
// whose chunks c1 .. w-1 sum to a log decay <= log_eps (the per-chunk sums of the WY step's
// summaries); -1 when the sum does not get there before the sequence end, or when one of those
// chunks breaks 0 <= beta |k|^2 <= 2.  A whole warp searches 32 chunks at a time; every lane returns
// the same.
__device__ __forceinline__ int rev_warmup_end(const float2* summ, int64_t bos, int n, int h, int Hv, int c1,
                                              int nck, float log_eps, int lane) {
    float cum = 0.f;
    bool bad = false;
    for (int bot = c1; bot < nck; bot += 32) {
        const int w = bot + lane;  // lane l looks at chunk bot + l
        const float2 cs = w < nck ? summ[img_slot(bos, n, w) * Hv + h] : make_float2(0.f, 0.f);
        float x = cs.x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, w < nck && cum + x <= log_eps);
        if (hit) {
            const int first = __ffs(hit) - 1;
            bad |= __any_sync(0xffffffffu, lane <= first && cs.y != 0.f);
            return bad ? -1 : bot + first + 1;
        }
        bad |= __any_sync(0xffffffffu, w < nck && cs.y != 0.f);
        cum += __shfl_sync(0xffffffffu, x, 31);
    }
    return -1;
}

// the adjoint scan's flags: 0 nothing yet, 1 the segment's fold (M, B) is published, 2 its exit
// adjoint is
__device__ __forceinline__ void rflag_release(int32_t* f, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ int rflag_acquire(const int32_t* f) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

__device__ __forceinline__ float bf(const uint8_t* tile, int row, int col) {  // bf16 element of a swizzled tile
    const uint8_t* p = tile + sw128_off(row, (col & 63) >> 3) + (col & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

// kPre: the adjoint scan's pre-pass, which runs before the reverse walk with the gradients on the
// same grid and runs the dH chain only.  A segment that takes the scan walks its own chunks twice,
// from dH = 0 (the fold B) and from dH = I with dO = 0 (the fold M), publishes the fold, looks
// forward for the nearest later segment whose exit adjoint is published, combines the folds in
// between (X <- M X + B, fp32) into its entry adjoint, which it records for its reverse walk, and
// publishes its own exit adjoint M X + B.  A segment that does not take the scan but has an
// earlier one that does walks to its exit adjoint from its usual start and publishes it.  Every
// other segment leaves at once.
// kPrep: the input preprocessing flags (GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM) are compiled in.
template <bool kPre, bool kPrep>
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
    float* red = (float*)(sm + bRed);        // [8 warps][32] partial sums
    float* acc_g = red + 256;                // dgamma accumulator [64]
    float* acc_b = red + 320;                // dbeta accumulator [64]
    float* acc_s = red + 384;                // scalars
    uint64_t* bar_ld = (uint64_t*)(sm + bBar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* tmem_slot = (uint32_t*)(bar_mma + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hv = p.Hv, dk = 128, dv = 128;
    const int glog = kPrep ? p.gate_logits : 0;  // GDN_FLAG_GATE_LOGITS, when compiled in
    // ---- which (sequence, head, segment) this CTA owns (the forward's scheme, except that the
    // later segments of a sequence take the lower block indices: a segment that takes the adjoint
    // scan waits for later ones, which are then scheduled no later than it)
    const int h = blockIdx.x % Hv;
    const int sidx = blockIdx.x / Hv;
    int n = 0, seg = 0, segs_n = 1;
    int64_t bos = 0, len = 0;
    if (!p.cu) {
        n = sidx / args.fixed_segs;
        segs_n = args.fixed_segs;
        seg = segs_n - 1 - sidx % args.fixed_segs;
        bos = (int64_t)n * p.T;
        len = p.T;
    } else {
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
                segs_n = __shfl_sync(0xffffffffu, s_m, src);
                seg = segs_n - 1 - (sidx - (base + __shfl_sync(0xffffffffu, incl - s_m, src)));
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
    // ---- reverse warm-up: walk later chunks from dH = 0 until their summed log decay is
    // <= log eps.  In a sequence of at least kRevScanMinSegs segments the adjoint scan takes over
    // where that fails, or where the warm-up would be longer than the scan's two fold walks over
    // the own chunks plus an allowance for the fold products (every such segment scans, so that
    // earlier ones find folds, not replays, between them and a published exit adjoint); else a
    // failed warm-up becomes a replay of the dH chain from dS_T at the sequence end.
    const bool scan_ok = args.scan_rec != nullptr && segs_n >= kRevScanMinSegs;
    auto takes_scan = [&](int c0j, int c1j, int wj) {
        return scan_ok && (wj < 0 || wj - c1j > 2 * (c1j - c0j) + kRevScanFoldAllowance);
    };
    int cend = nck;
    bool scan = false;
    if (c1 < nck && args.auto_warm) {
        const int w = rev_warmup_end(args.summ, bos, n, h, Hv, c1, nck, args.log_eps, lane);
        scan = takes_scan(c0, c1, w);
        if (w >= 0 && !scan) cend = w;
    }
    const bool exact_end = (cend == nck) && !scan;  // the walk starts from dS_T
    if constexpr (kPre) {
        // This segment's exit adjoint is published when an earlier segment of the sequence takes
        // the scan: the same decision, made here from the same summaries, one warp per earlier
        // segment.
        bool earlier_scans = false;
        if (scan_ok && args.auto_warm) {
            for (int j = seg - 1 - warp; j >= 0; j -= kNT / 32) {
                const int c0j = min(nck, j * args.L), c1j = min(nck, (j + 1) * args.L);
                if (c1j < nck &&
                    takes_scan(c0j, c1j, rev_warmup_end(args.summ, bos, n, h, Hv, c1j, nck, args.log_eps, lane)))
                    earlier_scans = true;
            }
        }
        if (!__syncthreads_or(earlier_scans) && !scan) {  // nothing to do in the pre-pass
            // (the pre-pass is a programmatic dependent of the state replay, which it does not read:
            // it completes only after the replay has, so that the reverse walk finds both done)
            asm volatile("griddepcontrol.wait;" ::: "memory");
            return;
        }
    }

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 2);  // one arrival per MMA issuer
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
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lane quarter
    const uint32_t sb = smem_u32(sm);
    // thread <-> TMEM lane m (an MMA row: a head-dimension index); the two warps of a lane
    // quarter split each row's columns (or tokens) in halves, hh = 0 / 1
    const int m = ((warp & 3) << 5) | lane;
    const int hh = warp >> 2;
    uint32_t ph_ld = 0, ph_mma = 0;
    bool ok = true;

    const uint32_t id_kk64 = idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mk64 = idesc_bf16(128, 64, 1, 0);
    const uint32_t id_km64 = idesc_bf16(128, 64, 0, 1);
    const uint32_t id_mm64 = idesc_bf16(128, 64, 1, 1);
    const uint32_t id_mm128 = idesc_bf16(128, 128, 1, 1);
    const uint32_t id_kk128 = idesc_bf16(128, 128, 0, 0);
    const uint32_t id_mk128 = idesc_bf16(128, 128, 1, 0);
    const float LOG2E = 1.4426950408889634f;

    // Two threads in different warps (0 and 32) issue the MMAs of a batch that write different
    // accumulators: one thread issues an N = 64 MMA about every 60 cycles, about twice the tensor
    // pipe's time for it, so two issuers finish a batch sooner.  Each commits its own MMAs to
    // bar_mma (two arrivals); a thread that issued none in a batch arrives directly.
    constexpr int kIss2 = 32;
    auto mma_sync_wait = [&](bool first, bool second) -> bool {
        if (tid == 0) {
            if (first) mma_commit(bar_mma);
            else mbar_arrive(bar_mma);
        }
        if (tid == kIss2) {
            if (second) mma_commit(bar_mma);
            else mbar_arrive(bar_mma);
        }
        const bool r = __syncthreads_and(mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
        tc_fence_after();
        return r;
    };
    // gates of chunk c: beta, gamma (cumsum), Gam, beta Gam, decay to the chunk end, E factors
    // g and beta of the next chunk in the walk, loaded one chunk ahead (threads 0..63)
    float nxt_g = 0.f, nxt_b = 0.f;
    auto prefetch_gates = [&](int c) {
        if (tid < 64 && c >= c0) {
            const int64_t t0 = bos + (int64_t)c * kChunk;
            const int lcc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
            // padding: g = beta = 0 (as raw gates: -inf, which the maps take to 0); raw gates are
            // mapped where they are used, a chunk later
            const float pad = glog ? -INFINITY : 0.f;
            nxt_g = tid < lcc ? p.g[(t0 + tid) * Hv + h] : pad;
            nxt_b = tid < lcc ? p.beta[(t0 + tid) * Hv + h] : pad;
        }
    };
    auto gates = [&](int c, int lc) -> bool {
        float gr = 0.f, gm = 0.f;
        if (tid < 64) {
            float x = gate_g(nxt_g, glog);
            const float bt = gate_beta(nxt_b, glog);
            prefetch_gates(c - 1);
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
    // E_rs for the 32 columns s0 .. s0 + 31 of row r: a_r b_s when every |gamma - gamma_31| < 80
    // (block-uniform), else exp2(a_r - b_s) with a = b = gamma log2(e)
    auto fill_E = [&](bool fac, int r, int s0, float* E) {
        const float ar = va[r];
        if (fac) {
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 b4 = *reinterpret_cast<const float4*>(vb + s0 + 4 * c4);
                E[4 * c4] = ar * b4.x;
                E[4 * c4 + 1] = ar * b4.y;
                E[4 * c4 + 2] = ar * b4.z;
                E[4 * c4 + 3] = ar * b4.w;
            }
        } else {
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 b4 = *reinterpret_cast<const float4*>(vb + s0 + 4 * c4);
                E[4 * c4] = exp2f(ar - b4.x);
                E[4 * c4 + 1] = exp2f(ar - b4.y);
                E[4 * c4 + 2] = exp2f(ar - b4.z);
                E[4 * c4 + 3] = exp2f(ar - b4.w);
            }
        }
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
    // Inputs of chunk c, all on bar_ld (one phase per chunk).  dO and the H image (chunks that
    // emit) are fetched as soon as the previous chunk in the walk has finished with their buffers
    // (after its [dP ; dA'] / H [dO ; TdU]^T products), v once its buffer has served as G there;
    // those fetches add their bytes to the phase without arriving.  q, k and the WY images follow
    // at the top of chunk c with the phase's one arrival.  The buffers' last generic reads and
    // writes were before the caller's barrier.
    auto load_do_h = [&](int c, bool with_h) {
        if (tid == 0) {
            const int t0 = (int)(bos + (int64_t)c * kChunk);
            fence_proxy_async();
            mbar_expect_tx(bar_ld, 16384 + (with_h ? kHImg : 0));  // dO: 2 x 8 KB (rows 0-63 of its tile)
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + bDO + a * 16384, &tm_do, bar_ld, 64 * a, h, t0);
            if (with_h) bulk_load(sm + bHt, args.himg + (img_slot(bos, n, c) * Hv + h) * kHImg, kHImg, bar_ld);
        }
    };
    auto load_v = [&](int c) {
        if (tid == 0) {
            const int t0 = (int)(bos + (int64_t)c * kChunk);
            fence_proxy_async();
            mbar_expect_tx(bar_ld, 16384);  // v: 2 x 8 KB
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + bV + a * 8192, &tm_v, bar_ld, 64 * a, h, t0);
        }
    };
    auto load_qk_wy = [&](int c) {
        if (tid == 0) {
            const int t0 = (int)(bos + (int64_t)c * kChunk);
            fence_proxy_async();
            mbar_arrive_expect_tx(bar_ld, 32768 + kWyImgBytes);  // q, k: 4 x 8 KB
            for (int a = 0; a < 2; ++a) {
                tma_load_3d(sm + bQK + a * 16384, &tm_q, bar_ld, 64 * a, hk, t0);
                tma_load_3d(sm + bQK + a * 16384 + 8192, &tm_k, bar_ld, 64 * a, hk, t0);
            }
            bulk_load(sm + bT, args.timg + (img_slot(bos, n, c) * Hv + h) * kWyImgBytes, kWyImgBytes, bar_ld);
        }
    };
    bool pre = false;  // dO, H and v of this chunk were fetched during the previous one
    // the scan's flag of segment j of this (sequence, value head), and its records
    auto flag_of = [&](int j) { return args.scan_flags + blockIdx.x + (int64_t)(seg - j) * Hv; };
    auto rec_of = [&](int j) {
        return args.scan_rec + (int64_t)(blockIdx.x + (int64_t)(seg - j) * Hv) * 4 * dk * dv;
    };
    // this CTA's records: [exit adjoint, M, B, entry adjoint], each [dk][dv]
    float* rec = args.scan_rec ? rec_of(seg) : nullptr;

    // ===================== reverse walk with the state adjoint =====================
    // One walk over the chunks (from dS_T, or from zero at the start of a reverse warm-up), or the
    // three walks of the adjoint scan over the own chunks: the fold B (from dH = 0), the fold M
    // (from dH = I with dO = 0), then the walk with the gradients from the scanned exit adjoint.
    {  // the walk's start: dS_T at the sequence end; for a segment that takes the scan, the entry
       // adjoint that the pre-pass recorded; zero at the start of a reverse warm-up (or of a fold)
        const float* src = nullptr;
        if (exact_end && b.dST) src = b.dST + ((int64_t)n * Hv + h) * dk * dv;
        if (!kPre && scan) src = rec + (int64_t)3 * dk * dv;
        float v[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] = src ? src[(int64_t)(64 * hh + e) * dv + m] : 0.f;
        tmem_st64(tl + cH + 64 * hh, v);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    // Walks: the reverse walk with the gradients (one walk); in the pre-pass the walk to the exit
    // adjoint (one walk, the dH chain only) or the two fold walks of the scan.
    auto run_walks = [&](auto walks) {
    constexpr int npass = decltype(walks)::value;
    for (int walk = 0; walk < npass && ok; ++walk) {
    const bool with_do = !(kPre && npass == 2 && walk == 1);  // the fold M has dO = 0
    const int ctop = scan ? c1 : cend;  // a walk covers chunks ctop - 1 down to c0
    prefetch_gates(ctop - 1);
    for (int c = ctop - 1; c >= c0 && ok; --c) {
        const bool emit = !kPre && c < c1;  // own chunk (else: warm-up or fold, the dH chain only)
        const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
        const int64_t t0 = bos + (int64_t)c * kChunk;
        // this chunk's inputs (first of all: their latency overlaps the copies and gates below)
        if (!pre) {
            load_do_h(c, emit);
            load_v(c);
        }
        load_qk_wy(c);
        pre = false;
        // bf16 copies of the exit adjoint dH_c: TMEM (A operand) and smem (MN-major A of dKd)
        {
            float v[64];
            uint32_t w[32];
            tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
            tmem_st32u(tl + cHb + 32 * hh, w);
            if (emit) {
                store_row32(sm + bDHt + hh * 16384, m, 0, v);
                store_row32(sm + bDHt + hh * 16384, m, 4, v + 32);
            }
        }
        if (tid < 64) {
            acc_g[tid] = 0.f;
            acc_b[tid] = 0.f;
        }
        if (tid < 8) acc_s[tid] = 0.f;
        const bool fac = gates(c, lc);
        ok = __syncthreads_and(mbar_wait(bar_ld, ph_ld));
        ph_ld ^= 1;
        if (!ok) break;
        if (kPrep && p.qk_norm)  // raw q and k rows (0-63 q, 64-127 k): normalised in place first
            l2norm_row_sw128(sm + bQK, 16384, tid >> 1, tid & 1);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        mma1();
        if (!(ok = mma_sync_wait(true, false))) break;
        // P (rows 0..63) -> smem
        if (m < 64) {  // P row m, this thread's half of the columns
            const int r = m;
            float v[32], E[32];
            tmem_ld32(tl + cR1 + 32 * hh, v);
            fill_E(fac, r, 32 * hh, E);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = 32 * hh + e;
                v[e] = (s <= r && r < lc) ? v[e] * E[e] : 0.f;
            }
            store_row32(sm + bP, r, 4 * hh, v);
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
        }
        if (tid == kIss2) {
            tc_fence_after();
            if (with_do) {
#pragma unroll
                for (int j = 0; j < 4; ++j)  // dO^T P (R4): A = dO^T MN-major, B = P MN-major (N = s)
                    mma_bf16_ss(tmem + cR4, desc_sw128(sb + bDO + j * 2048, 16384, 1024),
                                desc_sw128(sb + bP + j * 2048, 8192, 1024), id_mm64, j > 0);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // dH^T K^T (R5): A = bf16 dH^T (TMEM), B = K rows
                const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                mma_bf16_ts(tmem + cR5, tmem + cHb + 8 * j, desc_sw128(sb + bQK + 8192 + koff, 16, 1024),
                            id_kk64, j > 0);
            }
        }
        if (!(ok = mma_sync_wait(true, true))) break;
        {  // -W^T -> Wt;  Q rows * Gam -> Qg (over Bw/Bu);  dU^T -> bf16 (R5 cols 0..31);
           // <dH_c, H_c>, then dH^T <- Gam_n dH^T
            float v[64];
            tmem_ld32(tl + cR2 + 32 * hh, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = -v[e];
            store_row32(sm + bWt, m, 4 * hh, v);
            {
                // rows past the sequence end hold the next sequence's q and dO: zero them here
                // thread: row tid % 64 of dk half (tid / 64) % 2, 16-byte chunks 4 part .. 4 part + 3;
                // the eight lanes of a quarter warp take eight rows of one half (distinct banks)
                const int r = tid & 63, a = (tid >> 6) & 1, part = tid >> 7;
                const float gmul = r < lc ? vGam[r] : 0.f;
                const uint4* src = reinterpret_cast<const uint4*>(sm + bQK + a * 16384 + r * 128);
                uint4* dst = reinterpret_cast<uint4*>(sm + bBw + a * 8192 + r * 128);
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int c8 = (4 * part + i4 + r) & 7;
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
            {  // dU^T = dO^T P + (dH^T K^T) diag(dec) -> bf16 pairs in R5 columns 0..31; the other
               // half reads fp32 columns this half overwrites, hence the barrier
                float w32[32];
                tmem_ld32x2(tl + cR4 + 32 * hh, v, tl + cR5 + 32 * hh, w32);
                if (!with_do) {  // the fold of the linear part: dO = 0 (R4 was not written)
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0.f;
                }
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int s = 32 * hh + 2 * e;
                    w[e] = pack_bf16(v[2 * e] + vdec[s] * w32[2 * e], v[2 * e + 1] + vdec[s + 1] * w32[2 * e + 1]);
                }
                __syncthreads();
                tmem_st16u(tl + cR5 + 16 * hh, w);
            }
            float dhh = 0.f;
            const float Gn = vGam[63];
            tmem_ld64(tl + cH + 64 * hh, v);
            if (emit) {  // <dH_c, H_c> over this thread's row m, columns [64 hh, 64 hh + 64)
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint4 u = *reinterpret_cast<const uint4*>(sm + bHt + hh * 16384 + sw128_off(m, c8));
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        dhh += v[8 * c8 + 2 * e] * f.x + v[8 * c8 + 2 * e + 1] * f.y;
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] *= Gn;
            tmem_st64(tl + cH + 64 * hh, v);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dhh += __shfl_xor_sync(0xffffffffu, dhh, o);
            if (lane == 0) atomicAdd(&acc_s[0], dhh);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            if (emit) {
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
            }
        }
        if (tid == kIss2) {
            tc_fence_after();
            if (with_do) {
#pragma unroll
                for (int j = 0; j < 4; ++j)  // dH^T += dO^T Qg   (B = Qg MN-major, N = dk)
                    mma_bf16_ss(tmem + cH, desc_sw128(sb + bDO + j * 2048, 16384, 1024),
                                desc_sw128(sb + bBw + j * 2048, 8192, 1024), id_mm128, 1);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)  // dH^T += dU^T (-W)  (B = -W^T rows, K-major)
                mma_bf16_ts(tmem + cH, tmem + cR5 + 8 * j, desc_sw128(sb + bWt + j * 32, 16, 1024),
                            id_kk128, 1);
        }
        if (!(ok = mma_sync_wait(emit, true))) break;
        if (emit) {  // the chunk's gradients (own chunks only)
            {  // U^T -> Ut;  TdU: dv out, rows 64..127 of the dO tile, dbeta part;
               // this thread: row m of U^T and of TdU^T, tokens [32 hh, 32 hh + 32) in groups of 8
                __nv_bfloat16* dvp = (__nv_bfloat16*)b.dv + (t0 * Hv + h) * dv + (m & ~1);  // bf16 pairs
                const bool odd = m & 1;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    const int tb = 32 * hh + 8 * g;  // first token of the group
                    float u8[8], t8[8];
                    tmem_ld8x2(tl + cR3 + tb, u8, tl + cR2 + tb, t8);
                    *reinterpret_cast<uint4*>(sm + bUt + sw128_off(m, tb >> 3)) = pack8(u8);
                    const float4 bt0 = *reinterpret_cast<const float4*>(vbeta + tb);
                    const float4 bt1 = *reinterpret_cast<const float4*>(vbeta + tb + 4);
                    const float btv[8] = {bt0.x, bt0.y, bt0.z, bt0.w, bt1.x, bt1.y, bt1.z, bt1.w};
                    float bvals[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)  // TdU[r][m] v[r][m]
                        bvals[e] = t8[e] * bf(sm + bV + (m >> 6) * 8192, tb + e, m & 63);
                    // dv = beta TdU, and TdU into rows 64 + r of the stacked [dO ; TdU] tile, as bf16
                    // pairs (m & ~1, m | 1): lanes m, m^1 swap one value per two tokens, the even
                    // lane writes token tb + e, the odd one token tb + e + 1
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const float d0 = btv[e] * t8[e], d1 = btv[e + 1] * t8[e + 1];
                        const float rd = __shfl_xor_sync(0xffffffffu, odd ? d0 : d1, 1);
                        const float rt = __shfl_xor_sync(0xffffffffu, odd ? t8[e] : t8[e + 1], 1);
                        const int r = tb + e + (odd ? 1 : 0);
                        if (r < lc)
                            *reinterpret_cast<uint32_t*>(dvp + (int64_t)r * Hv * dv) =
                                odd ? pack_bf16(rd, d1) : pack_bf16(d0, rd);
                        *reinterpret_cast<uint32_t*>(sm + bDO + (m >> 6) * 16384 + sw128_off(64 + r, (m & 63) >> 3) +
                                                     (m & 6) * 2) = odd ? pack_bf16(rt, t8[e + 1]) : pack_bf16(t8[e], rt);
                    }
                    // sums over this warp's 32 m for each token: lane l ends with token tb + l / 4
                    warp_reduce_scatter<8>(bvals, lane);
                    bvals[0] += __shfl_xor_sync(0xffffffffu, bvals[0], 2);
                    bvals[0] += __shfl_xor_sync(0xffffffffu, bvals[0], 1);
                    if ((lane & 3) == 0) red[warp * 32 + 8 * g + (lane >> 2)] = bvals[0];
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            if (tid < 64) {
                const int q4 = (tid >> 5) * 4, l = tid & 31;
                acc_b[tid] += red[q4 * 32 + l] + red[(q4 + 1) * 32 + l] + red[(q4 + 2) * 32 + l] + red[(q4 + 3) * 32 + l];
            }
            if (tid == 0) {
                tc_fence_after();
    #pragma unroll
                for (int j = 0; j < 8; ++j) {  // [dP ; dA'] = [dO ; TdU] U^T   (R3): B = U^T MN-major
                    const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                    mma_bf16_ss(tmem + cR3, desc_sw128(sb + bDO + koff, 16, 1024),
                                desc_sw128(sb + bUt + j * 2048, 8192, 1024), id_km64, j > 0);
                }
    #pragma unroll
                for (int j = 0; j < 8; ++j)  // dKd^T = dH U^T (R2): A = dH (MN-major view of dH^T)
                    mma_bf16_ss(tmem + cR2, desc_sw128(sb + bDHt + j * 2048, 16384, 1024),
                                desc_sw128(sb + bUt + j * 2048, 8192, 1024), id_mm64, j > 0);
            }
            if (tid == kIss2) {
                tc_fence_after();
    #pragma unroll
                for (int j = 0; j < 8; ++j) {  // H [dO ; TdU]^T (R4 | R5, N = 128): A = H (MN-major view of
                                               // H^T), B = the stacked [dO ; TdU] rows; R4 = H dO^T and
                                               // R5 = H TdU^T = -TdW^T
                    const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                    mma_bf16_ss(tmem + cR4, desc_sw128(sb + bHt + j * 2048, 16384, 1024),
                                desc_sw128(sb + bDO + koff, 16, 1024), id_mk128, j > 0);
                }
            }
            if (!(ok = mma_sync_wait(true, true))) break;
            // the next chunk's dO and H image: this chunk's last reads of them were the products above
            pre = c - 1 >= c0;
            if (pre) load_do_h(c - 1, c - 1 < c1);
            {  // dP (lanes 0..63) and dA (lanes 64..127) rows, columns s in [32 hh, 32 hh + 32) in
               // four groups of eight: dgamma / dbeta terms, dP o E, G
                const int r = m & 63;
                const float ar = va[r], br = vbeta[r];
                float* G = (float*)(sm + bV);
                float rowsum = 0.f, bsum = 0.f;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    const int sb = 32 * hh + 8 * g;  // first column of the group
                    float d[8], x[8], E[8];
                    tmem_ld8x2(tl + cR3 + sb, d, tl + cR1 + sb, x);
                    {
                        const float4 b0 = *reinterpret_cast<const float4*>(vb + sb);
                        const float4 b1 = *reinterpret_cast<const float4*>(vb + sb + 4);
                        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        if (fac) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) E[e] = ar * bb[e];
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) E[e] = exp2f(ar - bb[e]);
                        }
                    }
                    // Outside the causal mask E may overflow (the decay factor of an entry above the
                    // diagonal is a growth factor): every product below uses E only through a
                    // select, so that no 0 * inf reaches the sums.
                    if (m < 64) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = sb + e;
                            const bool in = (s <= r && r < lc);
                            E[e] = in ? E[e] : 0.f;
                            const float P = in ? x[e] * E[e] : 0.f;
                            const float dP = in ? d[e] : 0.f;
                            rowsum += dP * P;
                            x[e] = dP * P;      // column-sum term
                            d[e] = dP * E[e];   // dP o E
                        }
                        *reinterpret_cast<uint4*>(sm + bP + sw128_off(r, sb >> 3)) = pack8(d);
                    } else {
                        float gw[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = sb + e;
                            const bool in = (s < r && r < lc);
                            E[e] = in ? E[e] : 0.f;
                            const float dA = in ? -d[e] : 0.f;
                            const float KE = x[e] * E[e];
                            const float A = br * KE;
                            rowsum += dA * A;
                            bsum += dA * KE;
                            x[e] = dA * A;
                            gw[e] = dA * E[e] * br;
                        }
                        *reinterpret_cast<float4*>(G + as_idx(r, sb)) = make_float4(gw[0], gw[1], gw[2], gw[3]);
                        *reinterpret_cast<float4*>(G + as_idx(r, sb + 4)) = make_float4(gw[4], gw[5], gw[6], gw[7]);
                    }
                    // column sums over this warp's rows: lane l ends with column sb + l / 4
                    warp_reduce_scatter<8>(x, lane);
                    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 2);
                    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
                    if ((lane & 3) == 0) red[warp * 32 + 8 * g + (lane >> 2)] = x[0];
                }
                // dgamma_r += rowsum (own row) - colsum (all rows) for both dP o P and dA o A
                atomicAdd(&acc_g[r], rowsum);
                if (m >= 64) atomicAdd(&acc_b[r], bsum);
                __syncthreads();
                if (tid < 64) {
                    const int q4 = (tid >> 5) * 4, l = tid & 31;
                    acc_g[tid] -= red[q4 * 32 + l] + red[(q4 + 1) * 32 + l] + red[(q4 + 2) * 32 + l] +
                                  red[(q4 + 3) * 32 + l];
                }
            }
            __syncthreads();
            {  // S = G + G^T, row s = tid % 64, columns [16 (tid / 64), + 16): G's rows as 16-byte
               // groups (as_idx keeps four columns together), its columns element by element
                const int s = tid & 63, qs = tid >> 6;
                const float* G = (const float*)(sm + bV);
                float v[16];
    #pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    const int j0 = 16 * qs + 4 * j4;
                    const float4 a = *reinterpret_cast<const float4*>(G + as_idx(s, j0));
                    v[4 * j4] = a.x + G[as_idx(j0, s)];
                    v[4 * j4 + 1] = a.y + G[as_idx(j0 + 1, s)];
                    v[4 * j4 + 2] = a.z + G[as_idx(j0 + 2, s)];
                    v[4 * j4 + 3] = a.w + G[as_idx(j0 + 3, s)];
                }
                *reinterpret_cast<uint4*>(sm + bT + sw128_off(s, 2 * qs)) = pack8(v);
                *reinterpret_cast<uint4*>(sm + bT + sw128_off(s, 2 * qs + 1)) = pack8(v + 8);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            if (pre) load_v(c - 1);  // G (over the v tile) has been read
            if (tid == 0) {
                tc_fence_after();
    #pragma unroll
                for (int j = 0; j < 4; ++j)  // dk^T main (R1): Q^T (dP o E) + K^T S^T
                    mma_bf16_ss(tmem + cR1, desc_sw128(sb + bQK + j * 2048, 16384, 1024),
                                desc_sw128(sb + bP + j * 2048, 8192, 1024), id_mm64, j > 0);
    #pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16_ss(tmem + cR1, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                                desc_sw128(sb + bT + j * 32, 16, 1024), id_mk64, 1);
            }
            if (tid == kIss2) {
                tc_fence_after();
    #pragma unroll
                for (int j = 0; j < 4; ++j)  // K^T (dP o E)^T (R3): A = K^T MN-major, B = dPE rows K-major
                    mma_bf16_ss(tmem + cR3, desc_sw128(sb + bQK + 8192 + j * 2048, 16384, 1024),
                                desc_sw128(sb + bP + j * 32, 16, 1024), id_mk64, j > 0);
            }
            if (!(ok = mma_sync_wait(true, true))) break;
            {  // epilogue: thread i = dk index (TMEM lane), tokens [32 hh, 32 hh + 32) in four
               // groups of eight (a rolled loop: a short body keeps the instruction stream small)
                const int i = m;
                float kdk = 0.f;
                const uint8_t* qtile = sm + bQK + (i >> 6) * 16384;
                // without grouped heads dq / dk go out directly (bf16); else per value head (fp32)
                // for the reduction over the group
                const bool direct = p.group == 1 && !(kPrep && p.qk_norm);
                float* dqp = args.dqw + (t0 * Hv + h) * dk + i;
                float* dkp = args.dkw + (t0 * Hv + h) * dk + i;
                __nv_bfloat16* dqb = (__nv_bfloat16*)b.dq + (t0 * Hv + h) * dk + (i & ~1);  // bf16 pairs
                __nv_bfloat16* dkb = (__nv_bfloat16*)b.dk + (t0 * Hv + h) * dk + (i & ~1);
                const bool odd = i & 1;
                float* red2 = (float*)(sm + bBw);  // [8 warps][32]: the Gam-scaled Q is no longer read
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    const int tb = 32 * hh + 8 * g;  // first token of the group
                    float hdo[8], kpe[8], dkm[8], dkd[8], tdw[8];
                    // H dO^T, K^T dPE^T, dk main, dKd^T, TdW^T for the group's 8 tokens
                    tmem_ld8x5(tl + cR4 + tb, hdo, tl + cR3 + tb, kpe, tl + cR1 + tb, dkm, tl + cR2 + tb, dkd,
                               tl + cR5 + tb, tdw);
#pragma unroll
                    for (int e = 0; e < 8; ++e) tdw[e] = -tdw[e];  // R5 holds H TdU^T = -TdW^T
                    float gam8[8], dec8[8], bg8[8];
#pragma unroll
                    for (int h4 = 0; h4 < 2; ++h4) {
                        const float4 x1 = *reinterpret_cast<const float4*>(vGam + tb + 4 * h4);
                        const float4 x2 = *reinterpret_cast<const float4*>(vdec + tb + 4 * h4);
                        const float4 x3 = *reinterpret_cast<const float4*>(vbG + tb + 4 * h4);
                        gam8[4 * h4] = x1.x; gam8[4 * h4 + 1] = x1.y; gam8[4 * h4 + 2] = x1.z; gam8[4 * h4 + 3] = x1.w;
                        dec8[4 * h4] = x2.x; dec8[4 * h4 + 1] = x2.y; dec8[4 * h4 + 2] = x2.z; dec8[4 * h4 + 3] = x2.w;
                        bg8[4 * h4] = x3.x; bg8[4 * h4 + 1] = x3.y; bg8[4 * h4 + 2] = x3.z; bg8[4 * h4 + 3] = x3.w;
                    }
                    float gv[8], bv[8], dq8[8], dk8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int r = tb + e;
                        const float qs = gam8[e] * hdo[e];  // dQs^T[i][r]
                        const float dqv = qs + kpe[e];
                        const float kv = bf(qtile, 64 + r, i & 63);
                        const float dkv = dkm[e] + dec8[e] * dkd[e] + bg8[e] * tdw[e];
                        dq8[e] = dqv;
                        dk8[e] = dkv;
                        if (!direct && r < lc) {
                            dqp[(int64_t)r * Hv * dk] = dqv;
                            dkp[(int64_t)r * Hv * dk] = dkv;
                        }
                        const float kdterm = dec8[e] * kv * dkd[e];
                        gv[e] = bf(qtile, r, i & 63) * qs + bg8[e] * tdw[e] * kv - kdterm;
                        bv[e] = gam8[e] * tdw[e] * kv;
                        kdk += kdterm;
                    }
                    if (direct) {  // bf16 pairs (i & ~1, i | 1): lanes i, i^1 swap one value per two tokens
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float sq = __shfl_xor_sync(0xffffffffu, odd ? dq8[e] : dq8[e + 1], 1);
                            const float sk = __shfl_xor_sync(0xffffffffu, odd ? dk8[e] : dk8[e + 1], 1);
                            const int r = tb + e + (odd ? 1 : 0);
                            if (r < lc) {
                                *reinterpret_cast<uint32_t*>(dqb + (int64_t)r * Hv * dk) =
                                    odd ? pack_bf16(sq, dq8[e + 1]) : pack_bf16(dq8[e], sq);
                                *reinterpret_cast<uint32_t*>(dkb + (int64_t)r * Hv * dk) =
                                    odd ? pack_bf16(sk, dk8[e + 1]) : pack_bf16(dk8[e], sk);
                            }
                        }
                    }
                    // sums over this warp's 32 i for each of the 8 tokens: lane l ends with token l / 4
                    warp_reduce_scatter<8>(gv, lane);
                    warp_reduce_scatter<8>(bv, lane);
                    gv[0] += __shfl_xor_sync(0xffffffffu, gv[0], 2);
                    gv[0] += __shfl_xor_sync(0xffffffffu, gv[0], 1);
                    bv[0] += __shfl_xor_sync(0xffffffffu, bv[0], 2);
                    bv[0] += __shfl_xor_sync(0xffffffffu, bv[0], 1);
                    if ((lane & 3) == 0) {
                        red[warp * 32 + 8 * g + (lane >> 2)] = gv[0];
                        red2[warp * 32 + 8 * g + (lane >> 2)] = bv[0];
                    }
                }
    #pragma unroll
                for (int o = 16; o > 0; o >>= 1) kdk += __shfl_xor_sync(0xffffffffu, kdk, o);
                if (lane == 0) atomicAdd(&acc_s[1], kdk);
                __syncthreads();
                if (tid < 64) {
                    const int q4 = (tid >> 5) * 4, l = tid & 31;
                    acc_g[tid] += red[q4 * 32 + l] + red[(q4 + 1) * 32 + l] + red[(q4 + 2) * 32 + l] +
                                  red[(q4 + 3) * 32 + l];
                    acc_b[tid] += red2[q4 * 32 + l] + red2[(q4 + 1) * 32 + l] + red2[(q4 + 2) * 32 + l] +
                                  red2[(q4 + 3) * 32 + l];
                }
                __syncthreads();
            }
            if (warp == 0) {  // last-row terms, then dg = reverse in-chunk cumsum of dgamma
                const float extra = acc_s[1] + vGam[63] * acc_s[0];
                const int r0 = 2 * lane;  // this lane's rows r0, r0 + 1
                const float x0 = r0 < lc ? acc_g[r0] + (r0 == lc - 1 ? extra : 0.f) : 0.f;
                const float x1 = r0 + 1 < lc ? acc_g[r0 + 1] + (r0 + 1 == lc - 1 ? extra : 0.f) : 0.f;
                float suf = x0 + x1;  // sum over the rows of lanes >= this one
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_down_sync(0xffffffffu, suf, o);
                    if (lane + o < 32) suf += y;
                }
                if (r0 < lc) b.dg[(t0 + r0) * Hv + h] = gate_g_grad(suf, glog ? p.g[(t0 + r0) * Hv + h] : 0.f, glog);
                if (r0 + 1 < lc)
                    b.dg[(t0 + r0 + 1) * Hv + h] = gate_g_grad(suf - x0, glog ? p.g[(t0 + r0 + 1) * Hv + h] : 0.f, glog);
            }
            if (tid < lc) b.dbeta[(t0 + tid) * Hv + h] = gate_beta_grad(acc_b[tid], vbeta[tid], glog);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (kPre && npass == 2 && ok && walk == 0) {
        // the fold B ended (from dH = 0): recorded [dk][dv] (thread (m, hh): dv column m, dk rows
        // [64 hh, 64 hh + 64)); the fold M starts from dH = I
        {
            float* dst = rec + (int64_t)2 * dk * dv + m;
            float v[64];
            tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
            for (int e = 0; e < 64; ++e) dst[(int64_t)(64 * hh + e) * dv] = v[e];
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = (64 * hh + e == m) ? 1.f : 0.f;
            tmem_st64(tl + cH + 64 * hh, v);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    }  // walks
    };
    if constexpr (kPre) {
        if (!scan) {
            run_walks(std::integral_constant<int, 1>{});  // to the exit adjoint, from the usual start
            if (ok) {
                float* ex = rec + m;
                float v[64];
                tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) ex[(int64_t)(64 * hh + e) * dv] = v[e];
                __threadfence();
                __syncthreads();
                if (tid == 0) rflag_release(flag_of(seg), 2);
            }
        } else {
            run_walks(std::integral_constant<int, 2>{});  // the folds B and M
        }
        if (scan && ok) {
            // the fold M (from dH = I with dO = 0), recorded; the fold is published
            {
                float* dst = rec + (int64_t)dk * dv + m;
                float v[64];
                tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) dst[(int64_t)(64 * hh + e) * dv] = v[e];
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) rflag_release(flag_of(seg), 1);
            // look forward: the nearest later segment whose exit adjoint is published (one that does
            // not take the scan publishes it after its walk; one that does, after its combination)
            int* lb = (int*)red;
            if (tid == 0) {
                int i = seg + 1;
                bool okl = true;
                const uint64_t tw = globaltimer();
                while (true) {
                    if (i >= segs_n) {  // no later segment published an exit adjoint
                        okl = false;
                        break;
                    }
                    const int f = rflag_acquire(flag_of(i));
                    if (f == 2) break;
                    if (f == 1) {
                        ++i;
                        continue;
                    }
                    if (globaltimer() - tw > kWaitTimeoutNs) {
                        okl = false;
                        break;
                    }
                    __nanosleep(128);
                }
                lb[0] = i;
                lb[1] = okl ? 1 : 0;
            }
            __syncthreads();
            ok = lb[1] != 0;
            const int base = lb[0];
            __syncthreads();  // lb has been read
            // X = the exit adjoint of segment base carried through the folds of segments base - 1 ..
            // seg, X <- M X + B, in fp32: before the own fold X is this segment's entry adjoint,
            // recorded for its reverse walk; after it, its exit adjoint.  Thread (m, hh) forms rows
            // [64 hh, 64 hh + 64) of column m from the whole column (both halves of TMEM lane m);
            // the exit record holds the new rows until both threads of the lane have read the old
            // column.
            float v[64];
            if (ok) {
                (void)rflag_acquire(flag_of(base));  // this thread's own acquire of the records it reads
                const float* ex = rec_of(base) + m;
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = ex[(int64_t)(64 * hh + e) * dv];
            } else {  // the look-forward timed out (reported): a zero entry adjoint, not garbage
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = 0.f;
                float* st = rec + (int64_t)3 * dk * dv + m;
#pragma unroll
                for (int e = 0; e < 64; ++e) st[(int64_t)(64 * hh + e) * dv] = 0.f;
            }
            tmem_st64(tl + cH + 64 * hh, v);
            float* tmp = rec + m;
            for (int t = base - 1; t >= seg && ok; --t) {
                (void)rflag_acquire(flag_of(t));
                tc_fence_before();
                __syncthreads();  // the column is complete in TMEM
                tc_fence_after();
                if (t == seg) {  // the entry adjoint of this segment's reverse walk
                    float* st = rec + (int64_t)3 * dk * dv + m;
                    tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
                    for (int e = 0; e < 64; ++e) st[(int64_t)(64 * hh + e) * dv] = v[e];
                }
                const float* Mt = rec_of(t) + dk * dv;
                const float* Bt = Mt + dk * dv;
#pragma unroll 1
                for (int ib = 0; ib < 2; ++ib) {  // rows 64 hh + 32 ib .. + 31 of the new column
                    const int r0 = 64 * hh + 32 * ib;
                    float acc[32];
#pragma unroll
                    for (int ii = 0; ii < 32; ++ii) acc[ii] = Bt[(int64_t)(r0 + ii) * dv + m];
#pragma unroll 1
                    for (int lb4 = 0; lb4 < 4; ++lb4) {  // times X rows 32 lb4 .. 32 lb4 + 31
                        float x[32];
                        tmem_ld32(tl + cH + 32 * lb4, x);
#pragma unroll 4
                        for (int ii = 0; ii < 32; ++ii) {
                            const float4* mr = reinterpret_cast<const float4*>(Mt + (int64_t)(r0 + ii) * dk + 32 * lb4);
                            float sacc = 0.f;
#pragma unroll
                            for (int l4 = 0; l4 < 8; ++l4) {
                                const float4 mv = mr[l4];
                                sacc += mv.x * x[4 * l4] + mv.y * x[4 * l4 + 1] + mv.z * x[4 * l4 + 2] +
                                        mv.w * x[4 * l4 + 3];
                            }
                            acc[ii] += sacc;
                        }
                    }
#pragma unroll
                    for (int ii = 0; ii < 32; ++ii) tmp[(int64_t)(r0 + ii) * dv] = acc[ii];
                }
                tc_fence_before();
                __syncthreads();  // both threads of every lane have read the old column
                tc_fence_after();
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = tmp[(int64_t)(64 * hh + e) * dv];
                tmem_st64(tl + cH + 64 * hh, v);
            }
            if (ok) {  // the exit adjoint M X + B is in the exit record: published
                __threadfence();
                __syncthreads();
                if (tid == 0) rflag_release(flag_of(seg), 2);
            }
        }
    } else {
        run_walks(std::integral_constant<int, 1>{});
    }
    if (!ok && pre) {  // fetches for the next chunk are in flight: let them land before the CTA exits
        if (tid == 0) mbar_arrive(bar_ld);
        (void)mbar_wait(bar_ld, ph_ld);
    }
    if (!kPre && ok && b.dS0 && seg == 0) {
        float* dst = b.dS0 + ((int64_t)n * Hv + h) * dk * dv + m;
        float v[64];
        tmem_ld64(tl + cH + 64 * hh, v);
#pragma unroll
        for (int e = 0; e < 64; ++e) dst[(int64_t)(64 * hh + e) * dv] = v[e];
    }
    if (!ok && tid == 0) report(p.status, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsB);
    }
    if constexpr (kPre) asm volatile("griddepcontrol.wait;" ::: "memory");  // see the early exit above
}


// The split of the reverse walks over CTAs, and whether some sequence has enough segments for the
// adjoint scan.  A reverse warm-up chunk runs only the dH chain: about a third of a full chunk.
struct RevSplit {
    std::vector<int> nck;
    SplitChoice sc;
    bool scan;
};

RevSplit rev_split(const Problem& p, const int32_t* cu_host, int split_mode) {
    RevSplit r;
    r.nck = chunk_counts(p, cu_host);
    r.sc = choose_split(r.nck, p.Hv, split_mode, sm_count(), 0.3);
    r.scan = false;
    for (int c : r.nck) r.scan |= segments_of(c, r.sc.L, 0) >= kRevScanMinSegs;
    r.scan &= split_mode != 1;
    return r;
}

// bytes of the adjoint scan's flags (one int32 per CTA, 256-aligned) and records (four fp32
// [dk][dv] states per CTA: exit adjoint, M, B, entry adjoint)
size_t rev_scan_flag_bytes(int64_t ctas) { return align_up((size_t)ctas * 4, 256); }
size_t rev_scan_bytes(const RevSplit& r, const Problem& p) {
    return r.scan ? rev_scan_flag_bytes(r.sc.ctas) + (size_t)r.sc.ctas * 4 * p.dk * p.dv * sizeof(float) : 0;
}

struct BwdLayout {
    size_t timg, himg, dqw, dkw, scan, total;
};

// workspace: the WY outputs (T / Bw / Bu images, gate summaries, the forward scan's flags and
// records), the replayed H^T images, (with grouped heads) fp32 dq and dk per value head, summed
// over each group by the reduction, then the adjoint scan's flags and records
BwdLayout bwd_layout(const Problem& p, const int32_t* cu_host, int split_mode) {
    BwdLayout l;
    size_t off = 0;
    l.timg = off;
    off = align_up(off + tc_fwd_workspace(p, cu_host, split_mode), 256);
    l.himg = off;
    off = align_up(off + (p.num_chunks > 0 ? (size_t)img_slots(p) * p.Hv * kHImg : 0), 256);
    // per-value-head fp32 dq / dk: summed over grouped heads, or taken through the chain rule of
    // the q / k normalisation, by the reduction kernel
    const size_t per = (p.group > 1 || p.qk_norm) ? sizeof(float) * (size_t)p.T_total * p.Hv * p.dk : 0;
    l.dqw = off;
    off = align_up(off + per, 256);
    l.dkw = off;
    off = align_up(off + per, 256);
    l.scan = off;
    off = align_up(off + (p.num_chunks > 0 ? rev_scan_bytes(rev_split(p, cu_host, split_mode), p) : 0), 256);
    l.total = off;
    return l;
}

}  // namespace

bool tc_bwd_supported(const Problem& p) { return p.dtype == GDN_BF16 && p.dk == 128 && p.dv == 128; }

size_t tc_bwd_workspace(const Problem& p, const int32_t* cu_host, int split_mode, size_t* off_himg,
                        size_t* off_timg, size_t* off_dqw, size_t* off_dkw) {
    const BwdLayout l = bwd_layout(p, cu_host, split_mode);
    *off_himg = l.himg;
    *off_timg = l.timg;
    *off_dqw = l.dqw;
    *off_dkw = l.dkw;
    return l.total;
}

int tc_bwd_launches(const Problem& p, const int32_t* cu_host, int split_mode) {
    if (p.num_chunks <= 0) return 1;
    // WY, state replay, [adjoint scan pre-pass,] reverse walk, [dq / dk group reduction]
    return 3 + (rev_split(p, cu_host, split_mode).scan ? 1 : 0) + ((p.group > 1 || p.qk_norm) ? 1 : 0);
}

gdn_status launch_bwd_tc(const BwdPlan& plan, char* ws, cudaStream_t s) {
    const BwdProblem& bp = plan.b;
    const Problem& p = bp.f;
    TcBwdArgs a;
    a.b = bp;
    const BwdLayout l = bwd_layout(p, plan.cu_host, plan.split_mode);
    const size_t oh = l.himg, ot = l.timg;
    a.himg = (const uint8_t*)(ws + oh);
    a.timg = (const uint8_t*)(ws + ot);
    a.summ = (const float2*)(ws + ot + wy_tc_summary_offset(p));
    a.dqw = (float*)(ws + l.dqw);
    a.dkw = (float*)(ws + l.dkw);
    const RevSplit rs = rev_split(p, plan.cu_host, plan.split_mode);
    const std::vector<int>& nck = rs.nck;
    const SplitChoice& sc = rs.sc;
    a.scan_flags = nullptr;
    a.scan_rec = nullptr;
    if (rs.scan && p.num_chunks > 0) {
        a.scan_flags = (int32_t*)(ws + l.scan);
        a.scan_rec = (float*)(ws + l.scan + rev_scan_flag_bytes(sc.ctas));
    }
    a.L = sc.L;
    a.fixed_segs = p.cu ? 0 : std::max(1, (nck.empty() ? 1 : (nck[0] + sc.L - 1) / sc.L));
    a.auto_warm = plan.split_mode == 1 ? 0 : 1;
    a.log_eps = (float)(-30.0 * std::log(2.0));
    CUtensorMap mq, mk, mv, mdo;
    const int64_t Tt = std::max<int64_t>(p.T_total, 1);
    if (!make_map(&mq, p.q, Tt, p.Hk) || !make_map(&mk, p.k, Tt, p.Hk) || !make_map(&mv, p.v, Tt, p.Hv) ||
        !make_map(&mdo, bp.dout, Tt, p.Hv))
        return GDN_ERR_CUDA;
    const bool prep = p.gate_logits || p.qk_norm;
    auto main_k = prep ? gdn_bwd_tc_kernel<false, true> : gdn_bwd_tc_kernel<false, false>;
    auto pre_k = prep ? gdn_bwd_tc_kernel<true, true> : gdn_bwd_tc_kernel<true, false>;
    if (cudaFuncSetAttribute(main_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemB) !=
            cudaSuccess ||
        (a.scan_rec &&
         cudaFuncSetAttribute(pre_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemB) !=
             cudaSuccess))
        return GDN_ERR_CUDA;
    if (sc.ctas > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (p.num_chunks > 0) {  // WY step + replay of the entry states
        // (its WY launch also clears the adjoint scan's flags)
        const gdn_status st = launch_replay_tc(p, plan.cu_host, plan.split_mode, ws + ot, (uint8_t*)(ws + oh), s,
                                               a.scan_flags, a.scan_flags ? (int)sc.ctas : 0);
        if (st) return st;
    }
    if (a.scan_rec) {
        // the adjoint scan's pre-pass on the same grid, as a programmatic dependent of the state
        // replay: it reads only the WY step's outputs (complete once every replay CTA has passed its
        // own wait for them), so its CTAs may run on the SMs the replay leaves free
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)sc.ctas);
        cfg.blockDim = dim3(kNT);
        cfg.dynamicSmemBytes = kSmemB;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, pre_k, mq, mk, mv, mdo, a) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    main_k<<<(unsigned)sc.ctas, kNT, kSmemB, s>>>(mq, mk, mv, mdo, a);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    if (p.T_total > 0 && (p.group > 1 || p.qk_norm)) return launch_bwd_reduce(bp, a.dqw, a.dkw, s);
    return GDN_OK;
}

}  // namespace gdn
