// gdn_decode.cu -- one recurrent (decode) step of the gated delta rule per (sequence, value
// head), applied to the state in place.  This is the step that follows a chunked prefill when
// a model generates token by token (news.hamidun.com "Qwen FlashQLA ... Hopper", scenario list:
// edge inference and distributed inference, several model calls in one stream); it consumes
// the S_T that gdn_chunk_fwd returns, in the same transposed layout H = S^T, [dk][dv].
//
// Per (sequence n, value head h), with H the state of slot s(n):
//   H <- exp(g) H,   p = H^T k,   H <- H + beta k (v - p)^T,   o = H^T q.
// Column j of H (a dv index) only meets k, q, v_j and the scalars, so with
//   a_j = H_old[:, j] . k,  b_j = H_old[:, j] . q,  d_j = beta (v_j - exp(g) a_j):
//   H_new[:, j] = exp(g) H_old[:, j] + d_j k,   o_j = exp(g) b_j + (k . q) d_j.
// The step is bound by HBM: each state (dk x dv fp32) is read once and written once.
//
// Kernel: one 256-thread CTA per (sequence, value head, 64 state columns): the columns of H never
// meet, so the state splits over CTAs by columns with no exchange.  Thread t owns the four
// columns 4 (t % 16) .. + 3 of its half and the rows t / 16, t / 16 + 16, ... (8 rows at
// dk = 128), so that half a warp reads and writes a 256-byte row piece with 16-byte accesses.
// The state piece goes into registers with all loads in flight at once (32 KB per CTA at
// d = 128), the two column dots are reduced over the 16 row groups in shared memory, and the new
// state is written back from registers: no thread reads a state element after another thread
// wrote it, so the update in place is safe, and different CTAs own different columns.  With 32
// state registers per thread (64 in all) four CTAs share an SM, so one CTA's loads overlap
// another's arithmetic and stores.
#include "gdn_dtype.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecCols = 64;                           // state columns per CTA
constexpr int kColGroups = kDecCols / 4;               // 16 (four columns per thread)
constexpr int kRowGroups = kDecThreads / kColGroups;   // 16
constexpr int kRowsPerThread = kMaxHead / kRowGroups;  // 8
constexpr int kDecMinBlocks = 4;  // CTAs per SM the registers are sized for (64 per thread)

struct DecodeArgs {
    int N, Hk, Hv, dk, dv, group, num_slots;
    const void* q;
    const void* k;
    const void* v;
    const float* beta;
    const float* g;
    float* S;
    const int32_t* idx;
    void* o;
    int32_t* status;
    int gate_logits;  // GDN_FLAG_GATE_LOGITS
    int qk_norm;      // GDN_FLAG_QK_L2NORM
};

// kPrep: the input preprocessing flags (GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM) are compiled in
template <typename Tin, bool kPrep>
__global__ void __launch_bounds__(kDecThreads, kDecMinBlocks) gdn_decode_kernel(const DecodeArgs a) {
    __shared__ float sk[kMaxHead], sq[kMaxHead], sv[kDecCols];
    __shared__ float4 pa[kRowGroups][kColGroups], pb[kRowGroups][kColGroups];  // partial column dots
    __shared__ float colA[kDecCols], colB[kDecCols];
    __shared__ float skq, sinv[2];
    const int h = blockIdx.x % a.Hv, n = blockIdx.x / a.Hv, hk = h / a.group;
    const int t = threadIdx.x, cg = t % kColGroups, rg = t / kColGroups;
    const int dk = a.dk, dv = a.dv;
    const int jb = kDecCols * blockIdx.y;  // this CTA's first state column
    const int slot = a.idx ? a.idx[n] : n;
    Tin* o = (Tin*)a.o + ((int64_t)n * a.Hv + h) * dv + jb;
    if (slot < 0) {  // padding entry of a batch: no state, zero output
        if (t < kDecCols && jb + t < dv) store_as(o + t, 0.f);
        return;
    }
    if (slot >= a.num_slots) {
        if (t == 0) report(a.status, GDN_ERR_DEVICE);
        return;
    }
    float* S = a.S + ((int64_t)slot * a.Hv + h) * dk * dv + jb;
    const bool col_ok = jb + 4 * cg < dv;

    // ---- the state into registers: every load issued before any is used
    float4 Hr[kRowsPerThread];
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = rg + kRowGroups * r;
        Hr[r] = (col_ok && i < dk) ? *reinterpret_cast<const float4*>(S + (int64_t)i * dv + 4 * cg)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const Tin* qp = (const Tin*)a.q + ((int64_t)n * a.Hk + hk) * dk;
    const Tin* kp = (const Tin*)a.k + ((int64_t)n * a.Hk + hk) * dk;
    const Tin* vp = (const Tin*)a.v + ((int64_t)n * a.Hv + h) * dv + jb;
    if (t < dk) {
        sk[t] = to_f(kp[t]);
        sq[t] = to_f(qp[t]);
    }
    if (t < kDecCols && jb + t < dv) sv[t] = to_f(vp[t]);
    const int glog = kPrep ? a.gate_logits : 0;
    const float eg = expf(gate_g(a.g[(int64_t)n * a.Hv + h], glog));
    const float bt = gate_beta(a.beta[(int64_t)n * a.Hv + h], glog);
    __syncthreads();
    if (kPrep && a.qk_norm) {  // raw k and q: x / max(|x|, eps), norms by warps 0 (k) and 1 (q)
        if (t < 64) {
            const float* x = t < 32 ? sk : sq;
            float ss = 0.f;
            for (int i = t & 31; i < dk; i += 32) ss += x[i] * x[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if ((t & 31) == 0) sinv[t >> 5] = 1.f / fmaxf(sqrtf(ss), kL2Eps);
        }
        __syncthreads();
        if (t < dk) {
            sk[t] *= sinv[0];
            sq[t] *= sinv[1];
        }
        __syncthreads();
    }
    if (t < 32) {  // k . q by warp 0
        float s = 0.f;
        for (int i = t; i < dk; i += 32) s += sk[i] * sq[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (t == 0) skq = s;
    }

    // ---- column dots a_j = H[:, j] . k and b_j = H[:, j] . q over this thread's rows
    float4 da = make_float4(0.f, 0.f, 0.f, 0.f), db = da;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = rg + kRowGroups * r;
        const float kk = i < dk ? sk[i] : 0.f, qq = i < dk ? sq[i] : 0.f;
        da.x += Hr[r].x * kk; da.y += Hr[r].y * kk; da.z += Hr[r].z * kk; da.w += Hr[r].w * kk;
        db.x += Hr[r].x * qq; db.y += Hr[r].y * qq; db.z += Hr[r].z * qq; db.w += Hr[r].w * qq;
    }
    pa[rg][cg] = da;
    pb[rg][cg] = db;
    __syncthreads();
    if (t < 2 * kColGroups) {  // sum the row groups: threads 0-15 for a, 16-31 for b
        const int c = t % kColGroups;
        const bool is_a = t < kColGroups;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < kRowGroups; ++g) {
            const float4 x = is_a ? pa[g][c] : pb[g][c];
            s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
        }
        float* dst = is_a ? colA : colB;
        if (jb + 4 * c < dv) *reinterpret_cast<float4*>(dst + 4 * c) = s;
    }
    __syncthreads();

    // ---- d_j, the new state, and the output
    if (!col_ok) return;
    float d[4], ob[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int j = 4 * cg + e;
        d[e] = bt * (sv[j] - eg * colA[j]);
        ob[e] = eg * colB[j] + skq * d[e];
    }
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = rg + kRowGroups * r;
        if (i < dk) {
            const float kk = sk[i];
            float4 w;
            w.x = eg * Hr[r].x + kk * d[0];
            w.y = eg * Hr[r].y + kk * d[1];
            w.z = eg * Hr[r].z + kk * d[2];
            w.w = eg * Hr[r].w + kk * d[3];
            *reinterpret_cast<float4*>(S + (int64_t)i * dv + 4 * cg) = w;
        }
    }
    if (rg == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) store_as(o + 4 * cg + e, ob[e]);
    }
}

}  // namespace

gdn_status plan_decode(const gdn_decode_args* a) {
    if (!a) return GDN_ERR_INVALID_ARG;
    if (a->struct_size < sizeof(gdn_decode_args) || a->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
    if (a->dtype != GDN_F32 && a->dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (a->N < 0 || a->Hk < 1 || a->Hv < 1 || a->Hv % a->Hk != 0) return GDN_ERR_INVALID_ARG;
    if (a->dk < 1 || a->dv < 1 || a->dk > kMaxHead || a->dv > kMaxHead || a->dv % 4 != 0)
        return GDN_ERR_UNSUPPORTED;
    const int64_t slots = a->state_indices ? (int64_t)a->num_slots : (int64_t)a->N;
    if (a->state_indices && a->num_slots < 1) return GDN_ERR_INVALID_ARG;
    if ((int64_t)a->N * a->Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (a->N == 0) return GDN_OK;
    const uintptr_t align16 = 15;
    if (!a->q || !a->k || !a->v || !a->beta || !a->g || !a->S || !a->o) return GDN_ERR_INVALID_ARG;
    if (((uintptr_t)a->S & align16) || ((uintptr_t)a->beta & 3) || ((uintptr_t)a->g & 3) ||
        ((uintptr_t)a->state_indices & 3) || ((uintptr_t)a->dev_status & 3))
        return GDN_ERR_INVALID_ARG;
    const size_t elt = a->dtype == GDN_BF16 ? 2 : 4;
    if (((uintptr_t)a->q | (uintptr_t)a->k | (uintptr_t)a->v | (uintptr_t)a->o) % elt)
        return GDN_ERR_INVALID_ARG;
    (void)slots;
    return GDN_OK;
}

gdn_status launch_decode(const gdn_decode_args* a, cudaStream_t s) {
    if (a->N == 0) return GDN_OK;
    DecodeArgs d;
    d.N = a->N;
    d.Hk = a->Hk;
    d.Hv = a->Hv;
    d.dk = a->dk;
    d.dv = a->dv;
    d.group = a->Hv / a->Hk;
    d.num_slots = a->state_indices ? a->num_slots : a->N;
    d.q = a->q;
    d.k = a->k;
    d.v = a->v;
    d.beta = a->beta;
    d.g = a->g;
    d.S = a->S;
    d.idx = a->state_indices;
    d.o = a->o;
    d.status = a->dev_status;
    d.gate_logits = (a->flags & GDN_FLAG_GATE_LOGITS) ? 1 : 0;
    d.qk_norm = (a->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    const dim3 grid((unsigned)((int64_t)a->N * a->Hv), (unsigned)((a->dv + kDecCols - 1) / kDecCols));
    const bool prep = d.gate_logits || d.qk_norm;
    if (a->dtype == GDN_BF16) {
        if (prep) gdn_decode_kernel<__nv_bfloat16, true><<<grid, kDecThreads, 0, s>>>(d);
        else gdn_decode_kernel<__nv_bfloat16, false><<<grid, kDecThreads, 0, s>>>(d);
    } else {
        if (prep) gdn_decode_kernel<float, true><<<grid, kDecThreads, 0, s>>>(d);
        else gdn_decode_kernel<float, false><<<grid, kDecThreads, 0, s>>>(d);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn

extern "C" gdn_status gdn_decode_step(const gdn_decode_args* args, void* stream) {
    using namespace gdn;
    const gdn_status st = plan_decode(args);
    if (st) return st;
    (void)cudaGetLastError();
    return launch_decode(args, (cudaStream_t)stream);
}
