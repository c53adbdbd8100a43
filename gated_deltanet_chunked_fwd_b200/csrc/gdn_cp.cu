// gdn_cp.cu -- the two device steps of context parallelism across GPUs for one long sequence
// whose tokens are sharded over several GPUs (dothoosh.com FlashQLA article, first innovation:
// gate-driven context parallelism, and its million-token paragraph).
//
// A shard of the sequence needs the state the sequence carries into it.  Every token maps the
// state affinely (H <- exp(g) (I - beta k k^T) H + beta k v^T in the H = S^T layout), so a shard
// maps its entry state as H_exit = M H_entry + B, and the entry state of shard r is the fold of
// shards 0..r-1 applied to S0:
//     X <- M_j X + B_j,  j = 0, 1, ..., r - 1                    (gdn_affine_combine)
// When the decay is strong the shard can instead start a few chunks early from a zero state:
// if the summed log decay over those halo tokens is <= log(eps) and every halo token keeps
// 0 <= beta |k|^2 <= 2 (so that each token's map has norm <= exp(g)), the truncated past
// changes the entry state by at most eps |H|                        (gdn_halo_check)
// The folds themselves are forward calls (B: S0 = 0; M: v = 0, S0 = [I | 0]); the collectives
// and the order of the steps are the caller's (the package's cp_chunk_fwd).
//
// Both kernels are small: the combine is dk x dk x dv fused multiply-adds per state (2.1 MFLOP
// at d = 128), the check reads the halo's k, beta and g once.
#include "gdn_dtype.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kCombThreads = 256;
constexpr int kCombCols = 32;                            // X columns per CTA (one per lane)
constexpr int kCombRowGroups = kCombThreads / kCombCols;  // 8 warps, rows strided by 8

// X <- M X + B for one state (blockIdx.x) and 32 of its columns (blockIdx.y).  The CTA reads its
// columns of X whole into shared memory before it writes any, and no other CTA touches them, so
// the update in place is safe.  Lane = column, warp = row group: a warp reads one M row element
// at a time (the same address in every lane: one broadcast) against 32 consecutive X columns.
__global__ void __launch_bounds__(kCombThreads) gdn_combine_kernel(const float* __restrict__ M,
                                                                   const float* __restrict__ B,
                                                                   float* __restrict__ X, int dk, int dv) {
    __shared__ float xs[kMaxHead][kCombCols + 1];
    const int64_t s = blockIdx.x;
    const int c0 = kCombCols * blockIdx.y;
    const int t = threadIdx.x, c = t % kCombCols, rg = t / kCombCols;
    const float* Ms = M + s * dk * dk;
    const float* Bs = B ? B + s * dk * dv : nullptr;
    float* Xs = X + s * dk * dv;
    const bool col = c0 + c < dv;
    for (int j = rg; j < dk; j += kCombRowGroups) xs[j][c] = col ? Xs[(int64_t)j * dv + c0 + c] : 0.f;
    __syncthreads();
    if (!col) return;
    for (int i = rg; i < dk; i += kCombRowGroups) {
        const float* mi = Ms + (int64_t)i * dk;
        float acc = 0.f;
        for (int j = 0; j < dk; ++j) acc = fmaf(mi[j], xs[j][c], acc);
        if (Bs) acc += Bs[(int64_t)i * dv + c0 + c];
        Xs[(int64_t)i * dv + c0 + c] = acc;
    }
}

struct HaloArgs {
    int T, Hk, Hv, dk, group;
    int gate_logits, qk_norm;
    float log_eps;
    const void* k;
    const float* beta;
    const float* g;
    int32_t* ok;
    float* log_decay;
};

constexpr int kHaloThreads = 256;

// One CTA per value head: each thread takes tokens t, t + 256, ...; the summed log decay and the
// norm condition are reduced over the CTA.
template <typename Tin>
__global__ void __launch_bounds__(kHaloThreads) gdn_halo_kernel(const HaloArgs a) {
    __shared__ float part[kHaloThreads / 32];
    const int h = blockIdx.x, hk = h / a.group;
    float sg = 0.f;
    bool bad = false;
    for (int t = threadIdx.x; t < a.T; t += kHaloThreads) {
        const float gt = gate_g(a.g[(int64_t)t * a.Hv + h], a.gate_logits);
        const float bt = gate_beta(a.beta[(int64_t)t * a.Hv + h], a.gate_logits);
        const Tin* kr = (const Tin*)a.k + ((int64_t)t * a.Hk + hk) * a.dk;
        float ss = 0.f;
        for (int i = 0; i < a.dk; ++i) {
            const float x = to_f(kr[i]);
            ss = fmaf(x, x, ss);
        }
        if (a.qk_norm) {  // |k / max(|k|, eps)|^2
            const float nrm = fmaxf(sqrtf(ss), kL2Eps);
            ss = ss / (nrm * nrm);
        }
        sg += gt;
        if (!(bt >= 0.f && bt * ss <= 2.f)) bad = true;  // also catches NaN
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sg += __shfl_xor_sync(0xffffffffu, sg, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sg;
    const bool any_bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        float sum = 0.f;
        for (int w = 0; w < kHaloThreads / 32; ++w) sum += part[w];
        a.ok[h] = (a.T > 0 && !any_bad && sum <= a.log_eps) ? 1 : 0;  // a NaN sum fails too
        if (a.log_decay) a.log_decay[h] = sum;
    }
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return a && b && na && nb && x < y + nb && y < x + na;
}

}  // namespace

gdn_status plan_combine(const gdn_combine_args* a) {
    if (!a) return GDN_ERR_INVALID_ARG;
    if (a->struct_size < sizeof(gdn_combine_args) || a->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
    if (a->N < 0 || a->Hv < 0) return GDN_ERR_INVALID_ARG;
    if (a->dk < 1 || a->dv < 1 || a->dk > kMaxHead || a->dv > kMaxHead) return GDN_ERR_UNSUPPORTED;
    const int64_t states = (int64_t)a->N * a->Hv;
    if (states > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (states == 0) return GDN_OK;
    if (!a->M || !a->X) return GDN_ERR_INVALID_ARG;
    if (((uintptr_t)a->M | (uintptr_t)a->B | (uintptr_t)a->X) & 15) return GDN_ERR_INVALID_ARG;
    const size_t nx = (size_t)states * a->dk * a->dv * 4, nm = (size_t)states * a->dk * a->dk * 4;
    if (overlaps(a->X, nx, a->M, nm) || overlaps(a->X, nx, a->B, nx)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status plan_halo(const gdn_halo_args* a) {
    if (!a) return GDN_ERR_INVALID_ARG;
    if (a->struct_size < sizeof(gdn_halo_args) || a->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
    if (a->dtype != GDN_F32 && a->dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (a->T < 0 || a->Hk < 1 || a->Hv < 1 || a->Hv % a->Hk != 0) return GDN_ERR_INVALID_ARG;
    if (a->dk < 1 || a->dk > kMaxHead) return GDN_ERR_UNSUPPORTED;
    if (a->Hv > 0x7fffffff / kHaloThreads) return GDN_ERR_UNSUPPORTED;
    if (!a->ok || ((uintptr_t)a->ok & 3) || ((uintptr_t)a->log_decay & 3)) return GDN_ERR_INVALID_ARG;
    if (a->T > 0) {
        if (!a->k || !a->beta || !a->g) return GDN_ERR_INVALID_ARG;
        const size_t elt = a->dtype == GDN_BF16 ? 2 : 4;
        if (((uintptr_t)a->k % elt) || ((uintptr_t)a->beta & 3) || ((uintptr_t)a->g & 3))
            return GDN_ERR_INVALID_ARG;
    }
    return GDN_OK;
}

gdn_status launch_combine(const gdn_combine_args* a, cudaStream_t s) {
    const int64_t states = (int64_t)a->N * a->Hv;
    if (states == 0) return GDN_OK;
    const dim3 grid((unsigned)states, (unsigned)((a->dv + kCombCols - 1) / kCombCols));
    gdn_combine_kernel<<<grid, kCombThreads, 0, s>>>(a->M, a->B, a->X, a->dk, a->dv);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_halo(const gdn_halo_args* a, cudaStream_t s) {
    HaloArgs h;
    h.T = a->T;
    h.Hk = a->Hk;
    h.Hv = a->Hv;
    h.dk = a->dk;
    h.group = a->Hv / a->Hk;
    h.gate_logits = (a->flags & GDN_FLAG_GATE_LOGITS) ? 1 : 0;
    h.qk_norm = (a->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    h.log_eps = a->log_eps;
    h.k = a->k;
    h.beta = a->beta;
    h.g = a->g;
    h.ok = a->ok;
    h.log_decay = a->log_decay;
    if (a->dtype == GDN_BF16) gdn_halo_kernel<__nv_bfloat16><<<a->Hv, kHaloThreads, 0, s>>>(h);
    else gdn_halo_kernel<float><<<a->Hv, kHaloThreads, 0, s>>>(h);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn

extern "C" gdn_status gdn_affine_combine(const gdn_combine_args* args, void* stream) {
    using namespace gdn;
    const gdn_status st = plan_combine(args);
    if (st) return st;
    (void)cudaGetLastError();
    return launch_combine(args, (cudaStream_t)stream);
}

extern "C" gdn_status gdn_halo_check(const gdn_halo_args* args, void* stream) {
    using namespace gdn;
    const gdn_status st = plan_halo(args);
    if (st) return st;
    (void)cudaGetLastError();
    return launch_halo(args, (cudaStream_t)stream);
}
