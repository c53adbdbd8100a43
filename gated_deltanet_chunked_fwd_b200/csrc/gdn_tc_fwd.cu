// gdn_tc_fwd.cu -- fused tensor-core forward of the chunked gated delta rule
// for bf16 tensors with dk = dv = 128 on sm_100a.
//
// Two launches do the whole forward.  The first (gdn_tc_wy.cu) forms, for every
// (chunk, value head) at once, the state-independent WY / UT inverse
// T = (I + A)^-1, A = strictly-lower(diag(beta) (K K^T o E)), and from it the bf16 images
// Bw = T diag(beta Gam) and Bu = T diag(beta) in the workspace.  The second (this file) is
// the fused state chain: each CTA owns one
// (sequence, value head, segment of chunks) and walks its chunks in order, keeping
// the fp32 state in TMEM; per chunk of C = 64 tokens (notation of gdn_internal.cuh):
//   gates      gamma = cumsum g, Gam, E = exp(gamma_r - gamma_s)       CUDA cores
//   MMA1       [Q;K] K^T -> Q K^T (rows 0-63 of the M=128 product)      tensor core
//   MMA_W/U    W^T = K^T Bw^T,  Ut^T = V^T Bu^T  (Bw, Bu: images of the WY step)
//   MMA_HW     U^T = Ut^T - H^T W^T  (accumulated onto Ut^T, B = -W^T)
//   MMA_O      O^T = H^T (diag(Gam) Q)^T + U^T P^T,  P = lower-incl(Q K^T o E)
//              (Q scaled by Gam in shared memory once Q K^T has read it; the outputs
//              are stored by the chunk-local warp group two chunks later)
//   MMA_H      H^T <- Gam_n H^T + (U^T diag(exp(gamma_n - gamma))) K
// All matrices are oriented so that a 128-wide head dimension is the MMA's M
// (TMEM lane = dv or dk index), so every MMA is M = 128 with N = 64 or 128.
// Operands live in shared memory as 128-byte-swizzled tiles; q / k / v tiles
// come in by TMA and the Bw / Bu images by a bulk copy (double-buffered: chunk c+2
// loads while chunks c and c+1 compute).
//
// Long sequences are split into segments that run on different SMs
// (gate-driven context parallelism, dothoosh.com FlashQLA article, first
// innovation): a segment that does not start its sequence starts from a zero
// state w chunks early, with w the fewest whole chunks whose summed log decay
// is <= log(eps).  While 0 <= beta |k|^2 <= 2 each token's state map has norm
// <= exp(g_t), so the truncated past contributes at most eps * |H| to the
// segment's entry state.  If the decay never reaches eps, or some warm-up
// token breaks the norm condition, the segment's entry state comes from an exact
// affine scan instead when that is cheaper than replaying the sequence from S0
// (long segments late in a sequence of at least scan_min_segs segments).  Every chunk maps the
// state affinely, H' = M_c H + B_c, so a segment's chunks compose to
// H_exit = M_j H_entry + B_j.  The segment folds (M_j, B_j) by walking its own
// chunks twice -- from H = 0 with the real values (B_j), then from H = I with
// v = 0 (M_j) -- and publishes them; it then looks back for the nearest earlier
// segment whose exit state is published (segments publish their exit when they
// end) and applies the folds in between, X <- M X + B, in fp32, which gives its
// exact entry state; a third walk from that state writes the outputs.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>
#include <cmath>
#include <vector>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"
#include "gdn_tc_common.cuh"


namespace gdn {

using namespace sm100;
using namespace tc;

namespace {

// Two groups of warps run a two-stage software pipeline over the chunks of a segment:
//   group P (threads 0-255, 8 warps)    chunk-local work of chunk k: the outputs of chunk k-2,
//                                       gates, Q K^T, P and diag(Gam) Q, W^T and Ut^T (Bw / Bu
//                                       images of the WY step as B operands), W^T -> smem
//   group S (threads 256-383, 4 warps)  the state chain of chunk k: U^T = Ut^T - H^T W^T,
//                                       O^T, H^T <- Gam_n H^T + (U^T diag(decay)) K, bf16 H
// Each group has a tcgen05 issuer (threads 0 and 256) and its own commit barrier; group P
// issues Ut^T from a second thread (kUIssuer, own barrier) at the same time as Q K^T, so that
// the two run together and only W^T waits for P.  The groups hand chunks over through
// mbarriers (full / empty pairs).  Warp w
// reads TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, so group P's two warps per lane
// quarter split the columns.
constexpr int kThreads = 384;
constexpr int kThreadsP = 256;
constexpr int kThreadsS = 128;
constexpr int kUIssuer = 96;  // group P's second MMA issuer (warp 3; thread 0 is the first)
constexpr int kTmemCols = 512;
// TMEM column map (lane = row of the M = 128 MMA)
constexpr uint32_t kColH = 0;     // H^T, fp32 state: lane dv, column dk     [0, 128)
constexpr uint32_t kColR1 = 128;  // Q K^T (lanes 0-63)                       [128, 192)
constexpr uint32_t kColR2 = 192;  // 2 x (Ut^T -> U^T), by chunk parity      [192, 320)
constexpr uint32_t kColO = 320;   // O^T = H^T (diag(Gam) Q)^T + U^T P^T        [320, 384)
constexpr uint32_t kColW = 384;   // W^T (group P)                              [384, 448)
constexpr uint32_t kColHb = 448;  // bf16 H^T, A operand (K pairs per column) [448, 512)
// U^T in bf16 (A operand of MMA_UP / MMA_H) overwrites the first 32 columns of its R2 buffer.

// shared memory carve-up (bytes from a 1024-aligned base)
constexpr uint32_t kStageQK = 0;       // 2 x 32 KB: [dk atom][q rows 0-63 | k rows 64-127][128 B]
constexpr uint32_t kStageV = 65536;    // 2 x 16 KB: [dv atom][64 rows][128 B]
constexpr uint32_t kPt = 98304;        // 2 x 8 KB  P: [64 n rows][64 s], by chunk parity
constexpr uint32_t kBwu = 114688;      // 2 x 16 KB  Bw = T diag(beta Gam), Bu = T diag(beta)
                                       // ([n][s] each, 8 KB apart), by chunk parity
constexpr uint32_t kWt = 147456;       // 16 KB  W^T: [128 dk rows][64 tokens]
constexpr uint32_t kVec = 163840;      // 4 x 2 KB of per-token vectors, by chunk index mod 4
constexpr uint32_t kVecStride = 512;   // floats per buffer
constexpr uint32_t kOst = kVec + 4 * kVecStride * 4;  // 16 KB bf16 o tile [dv atom][64 tokens][128 B]
constexpr uint32_t kRed = kOst + 16384;                // 16 floats
constexpr uint32_t kBar = kRed + 64;   // 10 mbarriers + TMEM base
constexpr uint32_t kSmemBytes = kBar + 128 + 1024;    // + alignment slack
static_assert(kBwu + 4 * kTImgBytes <= kWt && kWt + 16384 <= kVec, "shared-memory regions overlap");

struct TcArgs {
    Problem p;
    int L;          // chunks per segment
    int lead;       // extra chunks of a sequence's first segment (it needs no warm-up)
    int fixed_segs; // segments per sequence when cu_seqlens is absent
    int auto_warm;  // 1: gate-driven warm-up for segments that do not start a sequence
    float log_eps;  // warm-up stops once the summed log decay is <= log_eps
    const uint8_t* timg;  // T / Bw / Bu images of the WY step, by (image slot, value head)
    const float2* summ;   // per (image slot, value head): summed log decay, norm-condition flag
    uint8_t* himg;        // replay mode (backward): bf16 H^T entry-state image per own chunk, by
                          // (image slot, value head); no outputs.  nullptr: the forward
    // affine scan for segments that cannot warm up: per CTA (= blockIdx.x) a flag and three fp32
    // [dk][dv] records (exit state, M, B); nullptr (no sequence has scan_min_segs segments): such
    // a segment replays its sequence from S0 instead
    int32_t* scan_flags;
    float* scan_rec;
    int scan_min_segs;
};

// Warm-up start of the segment that begins at chunk c0 of sequence n (value head h): the largest
// w < c0 whose chunks w .. c0-1 sum to a log decay <= log_eps (the per-chunk sums of the WY step's
// summaries), searched 32 chunks at a time by a whole warp (every lane returns the same); -1 when
// the sum never gets there, or when one of those chunks breaks 0 <= beta |k|^2 <= 2.
__device__ __forceinline__ int warmup_start(const float2* summ, int64_t bos, int n, int h, int Hv, int c0,
                                            float log_eps, int lane) {
    float cum = 0.f;
    bool bad = false;
    for (int top = c0 - 1; top >= 0; top -= 32) {
        const int w = top - lane;  // lane l looks at chunk top - l
        const float2 cs = w >= 0 ? summ[img_slot(bos, n, w) * Hv + h] : make_float2(0.f, 0.f);
        float x = cs.x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, w >= 0 && cum + x <= log_eps);
        if (hit) {
            const int first = __ffs(hit) - 1;
            bad |= __any_sync(0xffffffffu, lane <= first && cs.y != 0.f);
            return bad ? -1 : top - first;
        }
        bad |= __any_sync(0xffffffffu, w >= 0 && cs.y != 0.f);
        cum += __shfl_sync(0xffffffffu, x, 31);
    }
    return -1;
}

// the scan's flags: 0 nothing yet, 1 the segment's fold (M, B) is published, 2 its exit state is
__device__ __forceinline__ void flag_release(int32_t* f, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ int flag_acquire(const int32_t* f) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

// Start state of the next walk of an affine scan, written to TMEM by the thread of state column m
// (lane m of the warp's quarter at tl): H = I when flags == nullptr; else the exit state of
// segment `base` (records at recs + base * stride: [exit, M, B], each [128][128] fp32, segments
// hv apart in the flags) carried through the folds of segments base + 1 .. seg - 1,
// X <- M X + B, in fp32; zero when base < 0 (a look-back that timed out).  The column of X lives
// in the fp32 state columns of TMEM while the folds run (32 x 32 blocks of M times 32 of its
// values at a time); `tmp` (this CTA's exit record) holds a fold's result column.  Ends with the
// bf16 copy in the A-operand columns and the fp32 state pre-scaled by Gn (the first chunk's Gam_n).
__device__ __forceinline__ void scan_start_state(uint32_t tl, int m, const int32_t* flags, int hv,
                                                 const float* recs, int64_t stride, int base, int seg,
                                                 float* tmp, float Gn) {
    constexpr int kD = 128;
    float v[32];
    if (!flags || base < 0) {
#pragma unroll 1
        for (int a = 0; a < 4; ++a) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = (flags == nullptr && 32 * a + e == m) ? 1.f : 0.f;
            tmem_st32(tl + kColH + 32 * a, v);
        }
    } else {
        (void)flag_acquire(flags + base * hv);  // this thread's own acquire of the records it reads
        const float* ex = recs + base * stride + m;
#pragma unroll 1
        for (int a = 0; a < 4; ++a) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = ex[(int64_t)(32 * a + e) * kD];
            tmem_st32(tl + kColH + 32 * a, v);
        }
        for (int t = base + 1; t < seg; ++t) {
            (void)flag_acquire(flags + t * hv);
            const float* Mt = recs + t * stride + kD * kD;
            const float* Bt = Mt + kD * kD;
#pragma unroll 1
            for (int ib = 0; ib < 4; ++ib) {  // rows 32 ib .. 32 ib + 31 of the new column
                float acc[32];
#pragma unroll
                for (int ii = 0; ii < 32; ++ii) acc[ii] = Bt[(int64_t)(32 * ib + ii) * kD + m];
#pragma unroll 1
                for (int lb = 0; lb < 4; ++lb) {  // times X rows 32 lb .. 32 lb + 31
                    tmem_ld32(tl + kColH + 32 * lb, v);
#pragma unroll 4
                    for (int ii = 0; ii < 32; ++ii) {
                        const float4* mr = reinterpret_cast<const float4*>(Mt + (int64_t)(32 * ib + ii) * kD + 32 * lb);
                        float sacc = 0.f;
#pragma unroll
                        for (int l4 = 0; l4 < 8; ++l4) {
                            const float4 mv = mr[l4];
                            sacc += mv.x * v[4 * l4] + mv.y * v[4 * l4 + 1] + mv.z * v[4 * l4 + 2] + mv.w * v[4 * l4 + 3];
                        }
                        acc[ii] += sacc;
                    }
                }
#pragma unroll
                for (int ii = 0; ii < 32; ++ii) tmp[(int64_t)(32 * ib + ii) * kD + m] = acc[ii];
            }
#pragma unroll 1
            for (int a = 0; a < 4; ++a) {  // the new column replaces X
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = tmp[(int64_t)(32 * a + e) * kD + m];
                tmem_st32(tl + kColH + 32 * a, v);
            }
        }
    }
    uint32_t w[16];
#pragma unroll 1
    for (int a = 0; a < 4; ++a) {
        tmem_ld32(tl + kColH + 32 * a, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        tmem_st16u(tl + kColHb + 16 * a, w);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= Gn;
        tmem_st32(tl + kColH + 32 * a, v);
    }
}

// kPrep: the input preprocessing flags (GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM) are compiled in;
// without them the kernel is the plain form.
template <bool kPrep>
__global__ void __launch_bounds__(kThreads, 1)
    gdn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const TcArgs args) {
    const Problem& p = args.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = (uint64_t*)(sm + kBar);
    uint64_t* bar_tma = bars;          // [2] stage full (TMA transaction bytes)
    uint64_t* bar_mma_p = bars + 2;    // warpgroup P's MMA completions
    uint64_t* bar_mma_s = bars + 3;    // warpgroup S's MMA completions
    uint64_t* bar_wt_full = bars + 4;  // W^T of chunk k in smem, Ut^T of chunk k in TMEM
    uint64_t* bar_wt_empty = bars + 5; // MMA_HW of chunk k has read W^T
    uint64_t* bar_s_done = bars + 6;   // [2] group S finished chunk k (parity buffers free)
    uint64_t* bar_mma_u = bars + 8;    // MMA_U and MMA_W completions (group P's second issuer)
    uint64_t* bar_o_free = bars + 9;   // group P has read chunk j's O^T out (arrival j)
    uint32_t* tmem_slot = (uint32_t*)(bars + 10);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
                s_m = max(1, (nchunks_of(l_m) - args.lead + args.L - 1) / args.L);
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
    // segment seg owns chunks [c0, c1): the first one [0, lead + L), then L each
    const int c0 = seg == 0 ? 0 : min(nck, args.lead + seg * args.L);
    const int c1 = min(nck, args.lead + (seg + 1) * args.L);

    // ---- set-up: barriers, TMEM
    if (tid == 0) {
        for (int i = 0; i < 10; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (!args.himg) prefetch_tensormap(&tm_o);
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

    // ---- initial state (warpgroup S): H^T (lane = dv index m) from S0 or zero
    auto load_state = [&](bool from_s0) {
        const int m = tid - kThreadsP;
        const float* s0 = (from_s0 && p.S0) ? p.S0 + ((int64_t)n * Hv + h) * dk * dv : nullptr;
        float v[64];
        uint32_t w[32];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
#pragma unroll
            for (int e = 0; e < 64; ++e) v[e] = s0 ? s0[(int64_t)(64 * a + e) * dv + m] : 0.f;
            tmem_st64(tl + kColH + 64 * a, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
            tmem_st32u(tl + kColHb + 32 * a, w);
        }
    };
    // A segment that starts its sequence (or any segment when the warm-up is off) starts
    // exactly from S0; that does not depend on the WY step, so it runs before waiting for it.
    const bool known_exact = (seg == 0) || !args.auto_warm;
    if (known_exact && tid >= kThreadsP) load_state(true);
    // The WY step (the previous launch) must be complete before its images and summaries are read.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // A programmatic dependent launch (the backward's adjoint-scan pre-pass, which reads the WY
    // step's outputs but not this grid's) may start once every CTA has passed the wait above.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- warm-up start (gate-driven); exact start from S0 when seg == 0.  The WY step left,
    // per chunk, its summed log decay and whether some token breaks 0 <= beta |k|^2 <= 2.
    // a segment without a warm-up takes the scan when its three walks over the own chunks and
    // one fold product per earlier segment (about three chunk steps each) cost less than
    // replaying the sequence's first chunks; else the replay from S0
    auto scan_pays = [&](int sj, int c0j, int c1j) {
        return args.scan_rec != nullptr && c0j > 2 * (c1j - c0j) + 3 * (sj - 1);
    };
    int cstart = 0;
    bool scan = false;  // entry state by the affine scan: three walks over the own chunks
    if (!known_exact) {
        const int w = warmup_start(args.summ, bos, n, h, Hv, c0, args.log_eps, lane);
        if (w < 0) {
            scan = scan_pays(seg, c0, c1);
            cstart = scan ? c0 : 0;
        } else {
            cstart = w;
        }
    }
    const bool exact = (cstart == 0);
    const int nkp = c1 - cstart;          // chunks per walk (warm-up + own)
    const int npass = scan ? 3 : 1;       // walks: [B fold, M fold,] final
    const int nk = npass * nkp;           // steps of the pipeline
    // step k of the pipeline: chunk cstart + k % nkp of walk k / nkp; walk 1 of a scan has v = 0
    auto chunk_of = [&](int k) {  // k < 3 nkp: two compares instead of a division
        int kk = k;
        if (kk >= nkp) kk -= nkp;
        if (kk >= nkp) kk -= nkp;
        return cstart + kk;
    };
    auto final_walk = [&](int k) { return k >= (npass - 1) * nkp; };
    auto v_on = [&](int k) { return !(scan && k >= nkp && k < 2 * nkp); };  // walk 1: v = 0
    // records of the scan, shared with the later segments of the sequence
    float* rec = args.scan_rec ? args.scan_rec + (int64_t)blockIdx.x * 3 * dk * dv : nullptr;
    if (!known_exact && tid >= kThreadsP) load_state(exact && !scan);
    auto issue_tma_at = [&](int k, int c) {  // step k, chunk c
        const int stage = k & 1;
        const int t0 = (int)(bos + (int64_t)c * kChunk);
        uint8_t* qk = sm + kStageQK + stage * 32768;
        uint8_t* vv = sm + kStageV + stage * 16384;
        mbar_arrive_expect_tx(&bar_tma[stage], 49152 + 2 * kTImgBytes);
        for (int a = 0; a < 2; ++a) {
            tma_load_3d(qk + a * 16384, &tm_q, &bar_tma[stage], 64 * a, hk, t0);
            tma_load_3d(qk + a * 16384 + 8192, &tm_k, &bar_tma[stage], 64 * a, hk, t0);
            tma_load_3d(vv + a * 8192, &tm_v, &bar_tma[stage], 64 * a, h, t0);
        }
        bulk_load(sm + kBwu + stage * 2 * kTImgBytes,
                  args.timg + (img_slot(bos, n, c) * Hv + h) * (int64_t)kWyImgBytes + kTImgBytes,
                  2 * kTImgBytes, &bar_tma[stage]);  // Bw and Bu
    };
    auto issue_tma = [&](int k) { issue_tma_at(k, chunk_of(k)); };

    if (tid == 0) {
        if (nk > 0) issue_tma(0);
        if (nk > 1) issue_tma(1);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t id_n64 = idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mn_n64 = idesc_bf16(128, 64, 1, 0);        // A MN-major
    const uint32_t id_bmn_n64 = idesc_bf16(128, 64, 0, 1);        // B MN-major
    const uint32_t id_bmn_n128 = idesc_bf16(128, 128, 0, 1);      // B MN-major, N = 128
    bool ok = true;

    if (tid < kThreadsP) {
        // ======================= group P: chunk-local work ======================
        const int t = tid;
        const int hf = t >> 7;                       // which 32-column half of a TMEM row
        const int row = ((warp & 3) << 5) | lane;    // TMEM lane (= MMA row) this thread reads
        uint32_t ph = 0;   // parity of bar_mma_p
        uint32_t phu = 0;  // parity of bar_mma_u
        // The loops come in two compiled forms: one walk over the chunks (every segment that does
        // not take the scan), or the three walks of the scan.
        auto run_p = [&](auto walks) {
        constexpr int NP = decltype(walks)::value;
        auto chunk_ofn = [&](int k) { return NP == 1 ? cstart + k : chunk_of(k); };
        auto final_walkn = [&](int k) { return NP == 1 || final_walk(k); };
        auto v_onn = [&](int k) { return NP == 1 || v_on(k); };
        // Gates run one chunk ahead in warp 2 (lane l: rows 2l, 2l+1), so chunk k+1's vectors
        // are in shared memory before chunk k is handed to group S.  g / beta of the chunk after
        // that are prefetched into registers.
        float gx0 = 0.f, gx1 = 0.f;
        const int glog = kPrep ? p.gate_logits : 0;  // GDN_FLAG_GATE_LOGITS, when compiled in
        auto load_gates = [&](int kk) {
            const int cc = chunk_ofn(kk);
            const int64_t t0 = bos + (int64_t)cc * kChunk;
            const int lcc = (int)min((int64_t)kChunk, len - (int64_t)cc * kChunk);
            const int r0 = 2 * lane;
            // padding: g = 0 (as a raw gate: -inf, which -softplus maps to 0); raw gates are mapped
            // where they are used, a chunk later, so that the prefetch does not wait here
            const float pad = glog ? -INFINITY : 0.f;
            gx0 = r0 < lcc ? p.g[(t0 + r0) * Hv + h] : pad;
            gx1 = r0 + 1 < lcc ? p.g[(t0 + r0 + 1) * Hv + h] : pad;
        };
        // vectors of chunk kk (buffer kk mod 4; beta enters through the Bw / Bu images): gamma =
        // cumsum g, Gam = exp(gamma), decay to the chunk end exp(gamma_n - gamma), the E factors
        // a, b, and the flag that says whether E_rs = a_r b_s (every |gamma - gamma_31| < 80) or
        // exp2(a_r - b_s)
        auto gates = [&](int kk) {
            float* vec = (float*)(sm + kVec) + (kk & 3) * kVecStride;
            const float m0 = gate_g(gx0, glog), m1 = gate_g(gx1, glog);
            float incl = m0 + m1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float g1 = incl, g0 = incl - m1;
            const float gm = __shfl_sync(0xffffffffu, g1, 15);  // gamma_31
            const float gl = __shfl_sync(0xffffffffu, g1, 31);  // gamma_63 (= gamma of the last token)
            const bool fac = __all_sync(0xffffffffu, fabsf(g0 - gm) < 80.f && fabsf(g1 - gm) < 80.f);
            const float LOG2E = 1.4426950408889634f;
            const float e0 = expf(g0), e1 = expf(g1);
            const int r0 = 2 * lane;
            *reinterpret_cast<float2*>(vec + 64 + r0) = make_float2(g0, g1);
            *reinterpret_cast<float2*>(vec + 128 + r0) = make_float2(e0, e1);
            *reinterpret_cast<float2*>(vec + 256 + r0) = make_float2(expf(gl - g0), expf(gl - g1));
            *reinterpret_cast<float2*>(vec + 320 + r0) =
                fac ? make_float2(expf(g0 - gm), expf(g1 - gm)) : make_float2(g0 * LOG2E, g1 * LOG2E);
            *reinterpret_cast<float2*>(vec + 384 + r0) =
                fac ? make_float2(expf(gm - g0), expf(gm - g1)) : make_float2(g0 * LOG2E, g1 * LOG2E);
            if (lane == 0) vec[448] = fac ? 1.f : 0.f;
        };
        if (warp == 2 && nk > 0) {
            load_gates(0);
            gates(0);
            if (nk > 1) load_gates(1);
        }
        // Outputs of chunk kk (once group S has finished it): o[t0+n][h][m] = O^T[m][n] from the
        // O^T buffer of parity kk; this warp covers dv rows 32 (warp & 3) .. + 31 and tokens
        // [32 hf, 32 hf + 32).  A whole chunk goes through a shared-memory tile and one TMA store
        // per 64-column half: the block is loaded in the 16x256b layout, whose registers form 8 x 8
        // matrix fragments (dv rows x tokens), and stmatrix stores them transposed, one 16-byte row
        // of 8 dv values per token.  A chunk cut short by its sequence's end is stored element by
        // element (this thread: dv row `row`), masked to its tokens.
        auto emits = [&](int kk) { return final_walkn(kk) && chunk_ofn(kk) >= c0 && !args.himg; };
        auto epilogue = [&](int kk) {
            const int cc = chunk_ofn(kk);
            const int64_t t0 = bos + (int64_t)cc * kChunk;
            const int lc = (int)min((int64_t)kChunk, len - (int64_t)cc * kChunk);
            // the last step's O^T goes to R1 (free by then), so that it need not wait for the read-out
            // of the step before
            const uint32_t colo = (kk == nk - 1 ? kColR1 : kColO) + 32 * hf;
            tc_fence_after();
            if (lc == kChunk) {
                const int j = lane >> 3, i = lane & 7;  // this lane addresses stored row i of matrix j
#pragma unroll
                for (int lh = 0; lh < 2; ++lh) {  // lane halves 0-15 and 16-31 of this warp's quarter
                    float f[16];
                    tmem_ld16x256b_x4(tl + ((uint32_t)(16 * lh) << 16) + colo, f);
                    if (lh == 0) {
                        if (t == 0) bulk_wait_read0();  // the previous chunk's store has read the tile
                        wg_sync(1, kThreadsP);
                    }
                    const int mrow = 32 * (warp & 3) + 16 * lh + 8 * (j & 1);  // first dv of its matrix
                    uint8_t* tile = sm + kOst + (mrow >> 6) * 8192;
#pragma unroll
                    for (int bp = 0; bp < 2; ++bp) {  // 8-token blocks 2 bp (matrices 0, 1), 2 bp + 1 (2, 3)
                        const float* r = f + 8 * bp;
                        const int token = 32 * hf + 8 * (2 * bp + (j >> 1)) + i;
                        stmatrix_x4_trans(smem_u32(tile + sw128_off(token, (mrow & 63) >> 3)),
                                          pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]),
                                          pack_bf16(r[6], r[7]));
                    }
                }
                fence_proxy_async();  // the tile is read by the TMA store
                tc_fence_before();    // O^T has been read (group S may overwrite it once told)
                wg_sync(1, kThreadsP);
                if (t == 0) {
                    tma_store_3d(&tm_o, sm + kOst, 0, h, (int)t0);
                    tma_store_3d(&tm_o, sm + kOst + 8192, 64, h, (int)t0);
                    bulk_commit();
                }
            } else {
                float ov[32];
                tmem_ld32(tl + colo, ov);
                __nv_bfloat16* op = (__nv_bfloat16*)p.o + (t0 * Hv + h) * dv + row;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int nn = 32 * hf + e;
                    if (nn < lc) op[(int64_t)nn * Hv * dv] = __float2bfloat16_rn(ov[e]);
                }
                tc_fence_before();
                wg_sync(1, kThreadsP);
            }
        };

        for (int k = 0; k < nk; ++k) {
            const int c = chunk_ofn(k);
            const int stage = k & 1;
            const bool emit = emits(k);
            const bool with_v = v_onn(k);  // walk 1 of a scan (the M fold) has v = 0: no Ut
            const int lc = (int)min((int64_t)kChunk, len - (int64_t)c * kChunk);
            const uint32_t sQK = sbase + kStageQK + stage * 32768;
            const uint32_t sV = sbase + kStageV + stage * 16384;
            const uint32_t sBwu = sbase + kBwu + stage * 2 * kTImgBytes;
            const float* vec = (const float*)(sm + kVec) + (k & 3) * kVecStride;
            const float* va = vec + 320;
            const float* vb = vec + 384;

            // buffers of parity `stage` are free once warpgroup S finished chunk k-2, whose
            // outputs are then final; group S writes the next O^T of this parity only after
            // this chunk's hand-off
            if (k >= 2) {
                ok = wg_and(1, kThreadsP, mbar_wait(&bar_s_done[stage], ((k - 2) >> 1) & 1));
                if (!ok) break;
                if (emits(k - 2)) epilogue(k - 2);
                if (t == 0) mbar_arrive(bar_o_free);  // arrival k - 2: O^T of chunk k - 2 is out
            }
            ok = wg_and(1, kThreadsP, mbar_wait(&bar_tma[stage], (k >> 1) & 1));
            if (!ok) break;
            if (kPrep && p.qk_norm) {  // raw q and k rows (0-63 q, 64-127 k): normalised in place first
                l2norm_row_sw128(sm + kStageQK + stage * 32768, 16384, t >> 1, t & 1);
                fence_proxy_async();
                wg_sync(1, kThreadsP);
            }
            if (emit && t == 0) {  // MMA1: [Q;K] K^T -> Q K^T (lanes 0-63; lanes 64-127 are unused);
                                   // a chunk without outputs (warm-up, fold walk, replay) needs none
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                    mma_bf16_ss(tmem + kColR1, desc_sw128(sQK + koff, 16, 1024),
                                desc_sw128(sQK + 8192 + koff, 16, 1024), id_n64, j > 0);
                }
                mma_commit(bar_mma_p);
            }
            if (t == kUIssuer) {  // MMA_U: Ut^T = V^T Bu^T (R2[stage]), unless the walk has v = 0, and
                                  // MMA_W: W^T = K^T Bw^T (its own columns), from a second issuer on
                                  // its own barrier while MMA1 runs
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (with_v)
                        mma_bf16_ss(tmem + kColR2 + 64 * stage, desc_sw128(sV + j * 2048, 8192, 1024),
                                    desc_sw128(sBwu + kTImgBytes + j * 32, 16, 1024), id_mn_n64, j > 0);
                    mma_bf16_ss(tmem + kColW, desc_sw128(sQK + 8192 + j * 2048, 16384, 1024),
                                desc_sw128(sBwu + j * 32, 16, 1024), id_mn_n64, j > 0);
                }
                mma_commit(bar_mma_u);
            }
            if (warp == 2 && k + 1 < nk) {  // the next chunk's gates, while MMA1 runs
                gates(k + 1);
                if (k + 2 < nk) load_gates(k + 2);
            }
            if (emit) {
                ok = wg_and(1, kThreadsP, mbar_wait(bar_mma_p, ph));
                ph ^= 1;
                if (!ok) break;
            }
            tc_fence_after();
            const bool fac = vec[448] != 0.f;

            // P (TMEM lanes 0..63: warps 0, 1, 4, 5, columns [32 hf, 32 hf + 32)) and, meanwhile,
            // Q rows <- Gam_n Q rows in place (warps 2, 3, 6, 7; MMA1 has read Q): the B operand
            // of MMA_O, so that H^T (diag(Gam) Q)^T and U^T P^T accumulate into one buffer
            if ((warp & 3) < 2) {
                if (emit) {
                    float v[32];
                    tmem_ld32(tl + kColR1 + 32 * hf, v);
                    const int r = row;
                    const int s0 = 32 * hf;
                    const float ar = va[r];
                    if (fac) {  // block-uniform: E_rs = a_r b_s
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4) {
                            const float4 b4 = *reinterpret_cast<const float4*>(vb + s0 + 4 * c4);
                            const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int s = s0 + 4 * c4 + e;
                                v[4 * c4 + e] = (s <= r && r < lc) ? v[4 * c4 + e] * (ar * bb[e]) : 0.f;
                            }
                        }
                    } else {  // E_rs = exp2(a_r - b_s) with a = b = gamma log2(e)
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4) {
                            const float4 b4 = *reinterpret_cast<const float4*>(vb + s0 + 4 * c4);
                            const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int s = s0 + 4 * c4 + e;
                                v[4 * c4 + e] = (s <= r && r < lc) ? v[4 * c4 + e] * exp2f(ar - bb[e]) : 0.f;
                            }
                        }
                    }
                    store_row32(sm + kPt + stage * 8192, r, 4 * hf, v);
                }
            } else if (emit) {
                const int li = ((warp >> 2) << 6) | ((warp & 1) << 5) | lane;  // 0..127
                const int srow = li >> 1;
                uint8_t* qrow = sm + kStageQK + stage * 32768 + (li & 1) * 16384 + srow * 128;
                const float gmul = vec[128 + srow];
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) {
                    const int c8 = (i8 + srow) & 7;  // rotated: rows spread over banks
                    uint4 u = *reinterpret_cast<uint4*>(qrow + 16 * c8);
                    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 f = __bfloat1622float2(b2[e2]);
                        b2[e2] = __floats2bfloat162_rn(f.x * gmul, f.y * gmul);
                    }
                    *reinterpret_cast<uint4*>(qrow + 16 * c8) = u;
                }
            }
            fence_proxy_async();  // Pt and diag(Gam) Q are read by the tensor core
            tc_fence_before();
            wg_sync(1, kThreadsP);

            {  // W^T and Ut^T are in TMEM, and Wt is free once MMA_HW of chunk k-1 has read it
                bool w = mbar_wait(bar_mma_u, phu);
                if (k >= 1) w = w && mbar_wait(bar_wt_empty, (k - 1) & 1);
                ok = wg_and(1, kThreadsP, w);
                phu ^= 1;
                if (!ok) break;
            }
            tc_fence_after();
            {  // W^T (lane = dk index) -> bf16 rows of the MN-major B operand of MMA_HW
                float v[32];
                tmem_ld32(tl + kColW + 32 * hf, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = -v[e];  // MMA_HW accumulates -H^T W^T
                store_row32(sm + kWt, row, 4 * hf, v);
            }
            fence_proxy_async();
            tc_fence_before();
            wg_sync(1, kThreadsP);
            if (t == 0) mbar_arrive(bar_wt_full);
        }
        for (int kk = max(nk - 2, 0); kk < nk && ok; ++kk) {  // the last two chunks' outputs
            ok = wg_and(1, kThreadsP, mbar_wait(&bar_s_done[kk & 1], (kk >> 1) & 1));
            if (ok && emits(kk)) epilogue(kk);
        }
        if (t == 0) bulk_wait0();  // every output tile has been written
        };
        if (npass == 1)
            run_p(std::integral_constant<int, 1>{});
        else
            run_p(std::integral_constant<int, 3>{});
    } else {
        // ======================= group S: the state chain =======================
        // Per chunk k: MMA_HW; U^T -> bf16 in TMEM; MMA_O (into the O^T buffer of the chunk's
        // parity, which group P reads out at chunk k+2) / MMA_H (A operands from TMEM); then one
        // pass over H that
        // writes its bf16 copy and pre-scales it by the next chunk's Gam_n (MMA_H of chunk
        // k+1 accumulates onto it).
        const int m = tid - kThreadsP;
        uint32_t ph = 0;  // parity of bar_mma_s
        // This segment's exit state is published when a later segment of the sequence takes the
        // scan: the same decision, made here from the same summaries, one warp per later segment
        // (while the first chunk is prepared by group P).
        bool later_scans = false;
        if (args.scan_rec != nullptr && args.auto_warm) {
            for (int j = seg + 1 + (warp & 3); j < segs_n; j += kThreadsS / 32) {
                const int c0j = min(nck, args.lead + j * args.L), c1j = min(nck, args.lead + (j + 1) * args.L);
                if (scan_pays(j, c0j, c1j) && warmup_start(args.summ, bos, n, h, Hv, c0j, args.log_eps, lane) < 0)
                    later_scans = true;
            }
        }
        const bool publish = wg_or(2, kThreadsS, later_scans);
        auto run_s = [&](auto walks) {
        constexpr int NP = decltype(walks)::value;
        auto issue_tman = [&](int k) {
            if (NP == 1) issue_tma_at(k, cstart + k);
            else issue_tma(k);
        };
        for (int walk = 0; walk < NP && ok; ++walk) {
        const bool fin = walk == NP - 1;       // the walk that writes outputs / entry images
        const bool with_v = NP == 1 || walk != 1; // walk 1 of a scan (the M fold) has v = 0
        for (int kk = 0; kk < nkp && ok; ++kk) {
            const int k = walk * nkp + kk;  // pipeline step
            const int c = cstart + kk;
            const int stage = k & 1;
            const bool emit = fin && c >= c0 && !args.himg;
            const uint32_t sQK = sbase + kStageQK + stage * 32768;
            const uint32_t colR2 = kColR2 + 64 * stage;
            const uint32_t colO = k == nk - 1 ? kColR1 : kColO;  // the last step's: R1 (group P is done with it)

            ok = wg_and(2, kThreadsS, mbar_wait(bar_wt_full, k & 1));
            if (!ok) break;
            if (k == 0) {
                // scale the initial state by Gam_n of the first chunk (its vectors were written
                // before the hand-off); MMA_H of chunk 0 accumulates onto it
                const float Gn = ((const float*)(sm + kVec))[128 + 63];
                float v[64];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    tmem_ld64(tl + kColH + 64 * a, v);
#pragma unroll
                    for (int e = 0; e < 64; ++e) v[e] *= Gn;
                    tmem_st64(tl + kColH + 64 * a, v);
                }
            }
            if (m == 0) {  // MMA_HW: U^T = Ut^T + H^T (-W^T)  (U^T = -H^T W^T when the walk has v = 0)
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    mma_bf16_ts(tmem + colR2, tmem + kColHb + 8 * j,
                                desc_sw128(sbase + kWt + j * 2048, 8192, 1024), id_bmn_n64, with_v || j > 0);
                mma_commit(bar_mma_s);
            }
            if (args.himg && c >= c0 && fin) {
                // replay mode: the chunk's entry state, as the bf16 H^T image [dk half][128 dv
                // rows][128 B] (128-byte swizzled) that the backward loads; the bf16 copy in TMEM
                // holds it (dk pairs per column).  Staged in the two 16 KB tiles that replay mode
                // leaves unused (P's tile and the output tile), then written by two bulk copies:
                // a thread per row writing 16 bytes into each of 128 rows straight to global
                // memory used only half of every sector it touched.
                uint8_t* img = args.himg + (img_slot(bos, n, c) * Hv + h) * (int64_t)32768;
                if (m == 0) bulk_wait_read0();  // the previous image's copies have read the tiles
                wg_sync(2, kThreadsS);
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    float w[32];
                    tmem_ld32(tl + kColHb + 32 * a, w);
                    uint8_t* tile = sm + (a == 0 ? kPt : kOst);
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4*>(tile + sw128_off(m, cc)) =
                            make_uint4(__float_as_uint(w[4 * cc]), __float_as_uint(w[4 * cc + 1]),
                                       __float_as_uint(w[4 * cc + 2]), __float_as_uint(w[4 * cc + 3]));
                }
                fence_proxy_async();  // the tiles are read by the bulk copies
                wg_sync(2, kThreadsS);
                if (m == 0) {
                    bulk_store(img, sm + kPt, 16384);
                    bulk_store(img + 16384, sm + kOst, 16384);
                    bulk_commit();
                }
            }
            ok = wg_and(2, kThreadsS, mbar_wait(bar_mma_s, ph));
            ph ^= 1;
            if (!ok) break;
            tc_fence_after();
            if (m == 0) mbar_arrive(bar_wt_empty);

            {  // U^T (lane = dv index, fp32) -> bf16 pairs in the same buffer: U^T in columns 0-31
               // (A of MMA_UP), U^T diag(exp(gamma_n - gamma)) in columns 32-63 (A of MMA_H)
                const float* vdec = (const float*)(sm + kVec) + (k & 3) * kVecStride + 256;
                float v[64];
                uint32_t w[32];
                tmem_ld64(tl + colR2, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
                tmem_st32u(tl + colR2, w);
#pragma unroll
                for (int e4 = 0; e4 < 16; ++e4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(vdec + 4 * e4);
                    w[2 * e4] = pack_bf16(v[4 * e4] * d4.x, v[4 * e4 + 1] * d4.y);
                    w[2 * e4 + 1] = pack_bf16(v[4 * e4 + 2] * d4.z, v[4 * e4 + 3] * d4.w);
                }
                tmem_st32u(tl + colR2 + 32, w);
            }
            tc_fence_before();
            // O^T of chunk k-1 has been read out by group P (its arrival k-1) before MMA_O rewrites
            // the buffer; chunks without outputs write none, and the last step writes R1
            ok = wg_and(2, kThreadsS, !(emit && k >= 1 && k < nk - 1) || mbar_wait(bar_o_free, (k - 1) & 1));
            if (!ok) break;
            if (m == 0) {  // MMA_O: O^T = H^T (diag(Gam) Q)^T + U^T P^T;  MMA_H: H^T += (U^T diag(decay)) K
                tc_fence_after();
                if (emit) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t koff = (j >> 2) * 16384 + (j & 3) * 32;
                        mma_bf16_ts(tmem + colO, tmem + kColHb + 8 * j, desc_sw128(sQK + koff, 16, 1024),
                                    id_n64, j > 0);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16_ts(tmem + colO, tmem + colR2 + 8 * j,
                                    desc_sw128(sbase + kPt + stage * 8192 + j * 32, 16, 1024), id_n64, 1);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16_ts(tmem + kColH, tmem + colR2 + 32 + 8 * j,
                                desc_sw128(sQK + 8192 + j * 2048, 16384, 1024), id_bmn_n128, 1);
                mma_commit(bar_mma_s);
            }
            ok = wg_and(2, kThreadsS, mbar_wait(bar_mma_s, ph));
            ph ^= 1;
            if (!ok) break;
            tc_fence_after();
            if (m == 0 && k + 2 < nk) issue_tman(k + 2);  // stage `stage` is no longer read

            // bf16 copy of the new state (A operand of the next chunk's MMAs); pre-scale by its Gam_n
            // (chunk k+1's vectors were written before chunk k was handed over).  The last chunk
            // of a fold walk leaves H as it is: the next walk starts from another state (below).
            const bool more = kk + 1 < nkp;
            {
                const float Gn = more ? ((const float*)(sm + kVec))[((k + 1) & 3) * kVecStride + 128 + 63] : 1.f;
                float v[64];
                uint32_t w[32];
#pragma unroll 1
                for (int a = 0; a < 2; ++a) {
                    tmem_ld64(tl + kColH + 64 * a, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
                    tmem_st32u(tl + kColHb + 32 * a, w);
                    if (more) {
#pragma unroll
                        for (int e = 0; e < 64; ++e) v[e] *= Gn;
                        tmem_st64(tl + kColH + 64 * a, v);
                    }
                }
            }
            tc_fence_before();
            wg_sync(2, kThreadsS);
            if (m == 0) mbar_arrive(&bar_s_done[stage]);
        }
        if (NP > 1 && ok && walk + 1 < NP) {
            // A fold walk ended: H is B_j (walk 0, from H = 0) or M_j (walk 1, from H = I with
            // v = 0); the next walk starts from I or from the scanned entry state.  Its first
            // chunk's vectors were written before the last chunk was handed over.
            tc_fence_after();
            const bool second = walk == 1;  // records of this CTA: [exit, M, B], each [dk][dv]
            {
                float* dst = rec + (int64_t)(second ? 1 : 2) * dk * dv + m;
                float v[64];
#pragma unroll 1
                for (int a = 0; a < 2; ++a) {
                    tmem_ld64(tl + kColH + 64 * a, v);
#pragma unroll
                    for (int e = 0; e < 64; ++e) dst[(int64_t)(64 * a + e) * dv] = v[e];
                }
            }
            const float Gn = ((const float*)(sm + kVec))[(((walk + 1) * nkp) & 3) * kVecStride + 128 + 63];
            if (!second) {
                scan_start_state(tl, m, nullptr, 0, nullptr, 0, 0, 0, nullptr, Gn);  // H = I
            } else {
                // publish the fold, then look back: the nearest earlier segment whose exit state
                // is published (segment 0 always publishes one), and the folds in between
                __threadfence();
                wg_sync(2, kThreadsS);
                int32_t* flags = args.scan_flags + (blockIdx.x - (unsigned)seg * Hv);  // segment 0
                if (m == 0) flag_release(flags + seg * Hv, 1);
                int* lb = (int*)(sm + kRed);
                if (m == 0) {
                    int i = seg - 1;
                    bool okl = true;
                    const uint64_t t0 = globaltimer();
                    while (true) {
                        const int f = flag_acquire(flags + i * Hv);
                        if (f == 2) break;
                        if (f == 1) {
                            --i;
                            continue;
                        }
                        if (globaltimer() - t0 > kWaitTimeoutNs) {
                            okl = false;
                            break;
                        }
                        __nanosleep(128);
                    }
                    lb[0] = i;
                    lb[1] = okl ? 1 : 0;
                }
                wg_sync(2, kThreadsS);
                ok = lb[1] != 0;
                const float* recs = args.scan_rec + (int64_t)(blockIdx.x - (unsigned)seg * Hv) * 3 * dk * dv;
                scan_start_state(tl, m, flags, Hv, recs, (int64_t)Hv * 3 * dk * dv, ok ? lb[0] : -1, seg, rec, Gn);
            }
            tc_fence_before();
            wg_sync(2, kThreadsS);
        }
        }  // walks
        };
        if (npass == 1)
            run_s(std::integral_constant<int, 1>{});
        else
            run_s(std::integral_constant<int, 3>{});
        if (ok && publish) {
            // the exit state for later segments that look back (the scan)
            float* ex = rec + m;
            float v[64];
#pragma unroll 1
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + kColH + 64 * a, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) ex[(int64_t)(64 * a + e) * dv] = v[e];
            }
            __threadfence();
            wg_sync(2, kThreadsS);
            if (m == 0) flag_release(args.scan_flags + blockIdx.x, 2);
        }
        if (ok && p.ST && seg == segs_n - 1) {
            // final state S_T = H (stored [dk][dv]): thread m writes column m
            float* st = p.ST + ((int64_t)n * Hv + h) * dk * dv + m;
            float v[64];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tmem_ld64(tl + kColH + 64 * a, v);
#pragma unroll
                for (int e = 0; e < 64; ++e) st[(int64_t)(64 * a + e) * dv] = v[e];
            }
        }
    }

    if (!ok && (tid == 0 || tid == kThreadsP)) report(p.status, GDN_ERR_TIMEOUT);
    if (args.himg && tid == kThreadsP) bulk_wait0();  // the entry-state images have been written
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------- host side
}  // namespace

bool tc_fwd_supported(const Problem& p) {
    return p.dtype == GDN_BF16 && p.dk == 128 && p.dv == 128;
}

namespace {

constexpr int kScanMinSegs = 4;  // the affine scan pays off from four segments on (three walks)

// The split of the chains over CTAs: the first segment of a sequence starts exactly, so it takes
// one chunk more than the others (a warm-up is at least one chunk).
struct ChainSplit {
    std::vector<int> nck;
    SplitChoice sc;
    bool scan;  // some sequence has enough segments for the affine scan
};

ChainSplit chain_split(const Problem& p, const int32_t* cu_host, int split_mode) {
    ChainSplit cs;
    cs.nck = chunk_counts(p, cu_host);
    cs.sc = choose_split(cs.nck, p.Hv, split_mode, sm_count(), 1.5, 1);
    cs.scan = false;
    for (int c : cs.nck) cs.scan |= segments_of(c, cs.sc.L, cs.sc.lead) >= kScanMinSegs;
    cs.scan &= split_mode != 1;
    return cs;
}

// bytes of the scan's flags (one int32 per CTA, 256-aligned) and records (three fp32 states
// [dk][dv] per CTA: exit state, M, B)
size_t scan_flag_bytes(int64_t ctas) { return align_up((size_t)ctas * 4, 256); }
size_t scan_bytes(const ChainSplit& cs, const Problem& p) {
    return cs.scan ? scan_flag_bytes(cs.sc.ctas) + (size_t)cs.sc.ctas * 3 * p.dk * p.dv * sizeof(float) : 0;
}

}  // namespace

// workspace: the T / Bw / Bu images and gate summaries of the WY step, then (when some sequence
// is split into enough segments) the affine scan's flags and records
size_t tc_fwd_workspace(const Problem& p, const int32_t* cu_host, int split_mode) {
    const size_t wy = align_up(wy_tc_workspace(p), 256);
    return p.num_chunks > 0 ? wy + scan_bytes(chain_split(p, cu_host, split_mode), p) : 0;
}
int tc_fwd_launches(const Problem& p) { return (p.num_chunks > 0 ? 1 : 0) + 1; }

// The WY kernel, then the fused kernel (forward, or replay of the states when himg != nullptr)
gdn_status launch_fwd_tc_impl(const Problem& p, const int32_t* cu_host, int split_mode, char* ws,
                              uint8_t* himg, cudaStream_t s, int32_t* rflags = nullptr, int nrflags = 0) {
    // all host-side preparation first, so that the two launches follow each other directly
    TcArgs a;
    a.p = p;
    a.timg = (const uint8_t*)ws;
    a.summ = (const float2*)(ws + wy_tc_summary_offset(p));
    a.himg = himg;
    const ChainSplit cs = chain_split(p, cu_host, split_mode);
    const std::vector<int>& nck = cs.nck;
    const SplitChoice& sc = cs.sc;
    a.scan_min_segs = kScanMinSegs;
    a.scan_flags = nullptr;
    a.scan_rec = nullptr;
    if (cs.scan && p.num_chunks > 0) {
        char* base = ws + align_up(wy_tc_workspace(p), 256);
        a.scan_flags = (int32_t*)base;
        a.scan_rec = (float*)(base + scan_flag_bytes(sc.ctas));
    }
    a.L = sc.L;
    a.lead = sc.lead;
    a.fixed_segs = p.cu ? 0 : (nck.empty() ? 1 : segments_of(nck[0], sc.L, sc.lead));
    a.auto_warm = split_mode == 1 ? 0 : 1;
    a.log_eps = (float)(-30.0 * std::log(2.0));
    CUtensorMap mq, mk, mv, mo;
    const int64_t Tt = std::max<int64_t>(p.T_total, 1);
    if (!make_map(&mq, p.q, Tt, p.Hk) || !make_map(&mk, p.k, Tt, p.Hk) || !make_map(&mv, p.v, Tt, p.Hv))
        return GDN_ERR_CUDA;
    // o (replay mode writes no o: the map is then never used)
    if (!make_map(&mo, p.o ? p.o : p.v, Tt, p.Hv)) return GDN_ERR_CUDA;
    auto kern = (p.gate_logits || p.qk_norm) ? gdn_fwd_tc_kernel<true> : gdn_fwd_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (sc.ctas > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    const gdn_status st =
        launch_wy_tc(p, mk, (uint8_t*)ws, a.scan_flags, a.scan_flags ? (int)sc.ctas : 0, rflags, nrflags,
                     himg != nullptr, s);
    if (st) return st;
    // Programmatic dependent launch: the fused kernel may start while the WY kernel drains; it
    // sets up and loads S0 for exact segments, then waits (griddepcontrol.wait) for the WY
    // kernel's outputs.  Only when the WY kernel is the previous launch in the stream, so that
    // nothing earlier (for instance the producer of S0) can overlap.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sc.ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.num_chunks > 0 ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, a) != cudaSuccess) return GDN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_fwd_tc(const FwdPlan& plan, char* ws, cudaStream_t s) {
    return launch_fwd_tc_impl(plan.p, plan.cu_host, plan.split_mode, ws, nullptr, s);
}

gdn_status launch_replay_tc(const Problem& p, const int32_t* cu_host, int split_mode, char* ws,
                            uint8_t* himg, cudaStream_t s, int32_t* rflags, int nrflags) {
    Problem q = p;  // states only: no o, no S_T
    q.o = nullptr;
    q.ST = nullptr;
    return launch_fwd_tc_impl(q, cu_host, split_mode, ws, himg, s, rflags, nrflags);
}

}  // namespace gdn
