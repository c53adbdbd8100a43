// gdn_tc_common.cuh -- pieces shared by the tensor-core forward and backward kernels:
// bf16 packing into 128-byte-swizzled shared-memory rows, the blocked fp32 triangular
// inverse T = (I + A)^-1 of a chunk (64 x 64), and the TMA tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

__device__ __forceinline__ int nchunks_of(int64_t len) { return (int)((len + kChunk - 1) / kChunk); }

// Per-(chunk, value head) images in the workspace are addressed by a slot: chunk c of
// sequence n, which starts at token bos, has slot floor(bos / 64) + n + c.  The WY step writes
// three bf16 64 x 64 tiles per (slot, value head), each 8 KB and 128-byte-swizzled [n][s]:
// T, then Bw = T diag(beta Gam), then Bu = T diag(beta).  Slots of different chunks never
// coincide (a sequence's chunks end at most one slot past floor(end / 64) + n, and the next
// sequence starts at floor(end / 64) + n + 1), and every slot is below img_slots().
constexpr uint32_t kTImgBytes = 8192;                // one 64 x 64 bf16 tile
constexpr uint32_t kWyImgBytes = 3 * kTImgBytes;     // T, Bw, Bu of one (slot, value head)
__host__ __device__ __forceinline__ int64_t img_slot(int64_t bos, int n, int c) {
    return bos / kChunk + n + c;
}
inline int64_t img_slots(const Problem& p) { return p.T_total / kChunk + p.N + 1; }

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

// group-wide barrier (named barrier `id` over `cnt` threads), plain and with an AND / OR vote
__device__ __forceinline__ void wg_sync(int id, int cnt) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(cnt) : "memory");
}
__device__ __forceinline__ bool wg_and(int id, int cnt, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(cnt)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool wg_or(int id, int cnt, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(cnt)
        : "memory");
    return r != 0;
}

// A (64 x 64, strictly lower) lives in As with float4 granules XOR-swizzled by row, so that a
// warp writing 32 rows at one column, or reading 8 rows at one column, hits distinct banks.
__device__ __forceinline__ int as_idx(int r, int s) { return r * 64 + ((((s >> 2) ^ (r & 15))) << 2) + (s & 3); }

// ------------------------------------------------------------------- host side
// Multi-SM split of the chunk chains (host side): chunks per sequence, and the segment length L
// that minimises the estimated makespan (waves of CTAs x chunk steps per CTA, a warm-up chunk
// counted as warm_cost steps).  split_mode: 0 auto, 1 off (one segment per sequence), 2 force (L = 2).
// GDN_FLAG_QK_L2NORM on a bf16 tile of 128-wide rows stored as two 64-column halves
// `half_bytes` apart, each row 128 bytes of 16-byte chunks swizzled by sw128_off: row `row` <-
// row / max(|row|_2, kL2Eps), with the sum of squares in fp32 and the result rounded to bf16 in
// place.  Two threads per row, adjacent lanes of one warp (`half` = 0 / 1, the lane's lowest
// bit): each reads, scales and writes its half; the two partial sums meet by one shuffle.  The
// caller orders the writes before the tensor core reads the tile (fence.proxy.async + barrier).
__device__ __forceinline__ void l2norm_row_sw128(uint8_t* tile, uint32_t half_bytes, int row, int half) {
    uint8_t* base = tile + half * half_bytes;
    float ss = 0.f;  // first pass: the sum of squares (the row is read twice to keep registers low)
#pragma unroll 2
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(base + sm100::sw128_off(row, c));
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(b2[e]);
            ss += f.x * f.x + f.y * f.y;
        }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    const float inv = 1.f / fmaxf(sqrtf(ss), kL2Eps);
#pragma unroll 2
    for (int c = 0; c < 8; ++c) {
        uint4 u = *reinterpret_cast<const uint4*>(base + sm100::sw128_off(row, c));
        __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(b2[e]);
            b2[e] = __floats2bfloat162_rn(f.x * inv, f.y * inv);
        }
        *reinterpret_cast<uint4*>(base + sm100::sw128_off(row, c)) = u;
    }
}

inline int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Segments of L chunks, except that the one segment of a sequence that starts exactly (it needs
// no warm-up) takes up to `lead` chunks more: a sequence of c chunks has
// max(1, ceil((c - lead) / L)) segments.  Count of CTAs over all sequences and value heads.
struct SplitChoice {
    int L;
    int lead;
    int64_t ctas;
};

inline int segments_of(int c, int L, int lead) { return std::max(1, (c - lead + L - 1) / L); }

// lead_auto: the exact segment's extra chunks in auto mode (0 keeps every segment at L)
inline SplitChoice choose_split(const std::vector<int>& nchunks, int Hv, int split_mode, int nsm,
                                double warm_cost = 1.5, int lead_auto = 0) {
    int maxc = 1;
    for (int c : nchunks) maxc = std::max(maxc, c);
    auto count = [&](int L, int lead) {
        int64_t s = 0;
        for (int c : nchunks) s += segments_of(c, L, lead);
        return s * Hv;
    };
    if (split_mode == 1) return {maxc, 0, count(maxc, 0)};
    if (split_mode == 2) {
        const int L = std::max(1, std::min(maxc, 2));
        return {L, 0, count(L, 0)};
    }
    int bestL = maxc, bestLead = 0;
    double best = 1e300;
    for (int L = 1; L <= maxc; ++L) {
        const int lead = L < maxc ? lead_auto : 0;
        const int64_t S = count(L, lead);
        const double waves = std::ceil((double)S / nsm);
        const double est = waves * (L + (L < maxc ? std::max(warm_cost, (double)lead) : 0.0));
        if (est < best - 1e-9 || (std::fabs(est - best) < 1e-9 && L > bestL)) {
            best = est;
            bestL = L;
            bestLead = lead;
        }
    }
    return {bestL, bestLead, count(bestL, bestLead)};
}

inline std::vector<int> chunk_counts(const Problem& p, const int32_t* cu_host) {
    std::vector<int> v;
    if (!p.cu) {
        v.assign(p.N, (p.T + kChunk - 1) / kChunk);
    } else {
        v.resize(p.N);
        for (int n = 0; n < p.N; ++n) v[n] = (cu_host[n + 1] - cu_host[n] + kChunk - 1) / kChunk;
    }
    return v;
}

// WY / UT step on its own: one bf16 T image per (chunk, value head), then per-chunk gate
// summaries, into the workspace `ws`; tm_k is k's tensor map (make_map below).  It also zeroes
// the nflags int32 flags of the state chain's affine scan and the nflags2 flags of the
// backward's adjoint scan (nullptr / 0: none).  The T image is
// written only when with_t (the backward reads it; the forward needs Bw and Bu).
gdn_status launch_wy_tc(const Problem& p, const CUtensorMap& tm_k, uint8_t* ws, int32_t* flags, int nflags,
                        int32_t* flags2, int nflags2, bool with_t, cudaStream_t s);

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder.  Calls may come from several host threads at once: the entry
// point is resolved once per process under std::call_once, and each calling thread first binds
// its device's primary context (once per thread), so that the driver call has a current context
// even in a thread whose first CUDA call this is.
inline EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    });
    thread_local bool bound = false;
    if (!bound) {
        int d = 0;
        bound = cudaGetDevice(&d) == cudaSuccess && cudaSetDevice(d) == cudaSuccess;
    }
    return fn;
}

// [T_total, H, 128] bf16 viewed as (d, head, token); box 64 x 1 x 64, 128-byte swizzle
inline bool make_map(CUtensorMap* map, const void* base, int64_t T_total, int H) {
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


}  // namespace tc
}  // namespace gdn
