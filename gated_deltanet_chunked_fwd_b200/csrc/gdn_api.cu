// gdn_api.cu -- the extern "C" entry points of libgdn.so: argument checks,
// planning, workspace carve-up and kernel dispatch.  Declarations and the
// contract (layouts, ownership, errors) are in include/gdn.h.
#include <string.h>

#include <climits>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr size_t kAlign = 256;

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

// Checks shared by forward and backward; fills the Problem (device pointers
// for outputs are filled by the callers).
gdn_status check_core(int dtype, int B, int T, int Hk, int Hv, int dk, int dv, int num_seqs,
                      const int32_t* cu, const int32_t* cu_host, Problem* p) {
    memset(p, 0, sizeof(*p));
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 1 || T < 0 || Hk < 1 || Hv < 1 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (dk < 1 || dv < 1 || dk > kMaxHead || dv > kMaxHead) return GDN_ERR_UNSUPPORTED;
    p->dtype = dtype;
    p->Hk = Hk;
    p->Hv = Hv;
    p->dk = dk;
    p->dv = dv;
    p->group = Hv / Hk;
    p->T = T;
    int64_t nc = 0;
    if (cu) {
        if (B != 1 || num_seqs < 1 || !cu_host) return GDN_ERR_INVALID_ARG;
        if (cu_host[0] != 0 || cu_host[num_seqs] != T) return GDN_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n) {
            if (cu_host[n + 1] < cu_host[n]) return GDN_ERR_INVALID_ARG;
            nc += (cu_host[n + 1] - cu_host[n] + kChunk - 1) / kChunk;
        }
        p->N = num_seqs;
        p->T_total = T;
        p->cu = cu;
    } else {
        p->N = B;
        p->T_total = (int64_t)B * T;
        nc = (int64_t)B * ((T + kChunk - 1) / kChunk);
    }
    if (p->T_total > INT_MAX || nc * Hv > INT_MAX) return GDN_ERR_UNSUPPORTED;
    p->num_chunks = nc;
    return GDN_OK;
}

gdn_status check_tensor(const void* ptr, bool needed, uintptr_t align) {
    if (!ptr) return needed ? GDN_ERR_INVALID_ARG : GDN_OK;
    return aligned(ptr, align) ? GDN_OK : GDN_ERR_INVALID_ARG;
}

// true when the byte ranges [a, a + n) and [b, b + n) share a byte (both non-NULL)
bool overlaps(const void* a, const void* b, size_t n) {
    if (!a || !b || n == 0) return false;
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + n && y < x + n;
}

// bytes of one state array [N, Hv, dk, dv] fp32
size_t state_bytes(const Problem& p) { return (size_t)p.N * p.Hv * p.dk * p.dv * sizeof(float); }

}  // namespace

gdn_status plan_fwd(const gdn_fwd_args* a, FwdPlan* plan) {
    if (!a || !plan) return GDN_ERR_INVALID_ARG;
    if (a->struct_size < sizeof(gdn_fwd_args) || a->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
    memset(plan, 0, sizeof(*plan));
    Problem& p = plan->p;
    gdn_status st = check_core(a->dtype, a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->num_seqs,
                               a->cu_seqlens, a->cu_seqlens_host, &p);
    if (st) return st;
    p.q = a->q;
    p.k = a->k;
    p.v = a->v;
    p.beta = a->beta;
    p.g = a->g;
    p.S0 = a->S0;
    p.o = a->o;
    p.ST = a->ST;
    p.status = a->dev_status;
    p.gate_logits = (a->flags & GDN_FLAG_GATE_LOGITS) ? 1 : 0;
    p.qk_norm = (a->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    plan->cu_host = a->cu_seqlens ? a->cu_seqlens_host : nullptr;
    plan->split_mode = (a->flags & GDN_FLAG_SPLIT_OFF) ? 1 : (a->flags & GDN_FLAG_SPLIT_FORCE) ? 2 : 0;
    plan->use_tc = !(a->flags & GDN_FLAG_PORTABLE) && tc_fwd_supported(p);
    const int64_t nc = p.num_chunks;
    size_t off = 0;
    if (plan->use_tc) {
        plan->total = align_up(tc_fwd_workspace(p, plan->cu_host, plan->split_mode), kAlign);
        plan->launches = tc_fwd_launches(p);
        return GDN_OK;
    }
    plan->off_table = off;
    off = align_up(off + sizeof(int32_t) * (3 * nc + p.N + 1), kAlign);
    plan->off_W = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk * p.dk, kAlign);
    plan->off_U = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk * p.dv, kAlign);
    plan->off_gam = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk, kAlign);
    plan->off_Hc = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * p.dk * p.dv, kAlign);
    plan->total = off;
    plan->launches = nc > 0 ? 4 : 2;
    return GDN_OK;
}

static gdn_status check_fwd_pointers(const gdn_fwd_args* a, const Problem& p) {
    const bool any = p.T_total > 0;
    gdn_status st;
    if ((st = check_tensor(a->q, any, 16)) || (st = check_tensor(a->k, any, 16)) ||
        (st = check_tensor(a->v, any, 16)) || (st = check_tensor(a->o, any, 16)) ||
        (st = check_tensor(a->beta, any, 4)) || (st = check_tensor(a->g, any, 4)) ||
        (st = check_tensor(a->S0, false, 16)) || (st = check_tensor(a->ST, false, 16)) ||
        (st = check_tensor(a->dev_status, false, 4)) || (st = check_tensor(a->cu_seqlens, false, 4)))
        return st;
    // S0 and S_T must not share memory: a segment of a split sequence may read S0 after the
    // sequence's last segment (another CTA) has written S_T
    if (overlaps(a->S0, a->ST, state_bytes(p))) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status plan_bwd(const gdn_bwd_args* a, BwdPlan* plan) {
    if (!a || !plan) return GDN_ERR_INVALID_ARG;
    if (a->struct_size < sizeof(gdn_bwd_args) || a->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
    memset(plan, 0, sizeof(*plan));
    Problem& p = plan->b.f;
    gdn_status st = check_core(a->dtype, a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->num_seqs,
                               a->cu_seqlens, a->cu_seqlens_host, &p);
    if (st) return st;
    p.q = a->q;
    p.k = a->k;
    p.v = a->v;
    p.beta = a->beta;
    p.g = a->g;
    p.S0 = a->S0;
    p.status = a->dev_status;
    p.gate_logits = (a->flags & GDN_FLAG_GATE_LOGITS) ? 1 : 0;
    p.qk_norm = (a->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    BwdProblem& b = plan->b;
    b.dout = a->dout;
    b.dST = a->dST;
    b.dq = a->dq;
    b.dk = a->dk_out;
    b.dv = a->dv_out;
    b.dbeta = a->dbeta;
    b.dg = a->dg;
    b.dS0 = a->dS0;
    const int64_t nc = p.num_chunks;
    plan->use_tc = !(a->flags & GDN_FLAG_PORTABLE) && tc_bwd_supported(p);
    plan->cu_host = a->cu_seqlens ? a->cu_seqlens_host : nullptr;
    plan->split_mode = (a->flags & GDN_FLAG_SPLIT_OFF) ? 1 : (a->flags & GDN_FLAG_SPLIT_FORCE) ? 2 : 0;
    if (plan->use_tc) {
        size_t o1, o2, o3, o4;
        plan->total = align_up(tc_bwd_workspace(p, plan->cu_host, plan->split_mode, &o1, &o2, &o3, &o4), kAlign);
        plan->launches = tc_bwd_launches(p, plan->cu_host, plan->split_mode);
        return GDN_OK;
    }
    size_t off = 0;
    plan->off_table = off;
    off = align_up(off + sizeof(int32_t) * (3 * nc + p.N + 1), kAlign);
    plan->off_W = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk * p.dk, kAlign);
    plan->off_U = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk * p.dv, kAlign);
    plan->off_gam = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk, kAlign);
    plan->off_Hc = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * p.dk * p.dv, kAlign);
    plan->off_dHc = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * p.dk * p.dv, kAlign);
    plan->off_dU = off;
    off = align_up(off + sizeof(float) * nc * p.Hv * kChunk * p.dv, kAlign);
    plan->off_dqw = off;
    off = align_up(off + sizeof(float) * p.T_total * p.Hv * p.dk, kAlign);
    plan->off_dkw = off;
    off = align_up(off + sizeof(float) * p.T_total * p.Hv * p.dk, kAlign);
    plan->total = off;
    plan->launches = nc > 0 ? 6 : 2;
    return GDN_OK;
}

static gdn_status check_bwd_pointers(const gdn_bwd_args* a, const Problem& p) {
    const bool any = p.T_total > 0;
    gdn_status st;
    if ((st = check_tensor(a->q, any, 16)) || (st = check_tensor(a->k, any, 16)) ||
        (st = check_tensor(a->v, any, 16)) || (st = check_tensor(a->dout, any, 16)) ||
        (st = check_tensor(a->beta, any, 4)) || (st = check_tensor(a->g, any, 4)) ||
        (st = check_tensor(a->dq, any, 16)) || (st = check_tensor(a->dk_out, any, 16)) ||
        (st = check_tensor(a->dv_out, any, 16)) || (st = check_tensor(a->dbeta, any, 4)) ||
        (st = check_tensor(a->dg, any, 4)) || (st = check_tensor(a->S0, false, 16)) ||
        (st = check_tensor(a->dST, false, 16)) || (st = check_tensor(a->dS0, false, 16)) ||
        (st = check_tensor(a->dev_status, false, 4)) || (st = check_tensor(a->cu_seqlens, false, 4)))
        return st;
    // dS0 is written while other CTAs may still read S0 (state replay) or dS_T (segments that
    // start their reverse walk exactly): no shared memory between them
    const size_t sb = state_bytes(p);
    if (overlaps(a->dS0, a->S0, sb) || overlaps(a->dS0, a->dST, sb)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

static gdn_status check_workspace(void* ws, size_t bytes, size_t need) {
    if (need == 0) return GDN_OK;
    if (!ws || bytes < need || !aligned(ws, kAlign)) return GDN_ERR_WORKSPACE;
    return GDN_OK;
}

}  // namespace gdn

using namespace gdn;

extern "C" {

gdn_status gdn_chunk_fwd_workspace_size(const gdn_fwd_args* args, size_t* bytes) {
    if (!bytes) return GDN_ERR_INVALID_ARG;
    FwdPlan plan;
    gdn_status st = plan_fwd(args, &plan);
    if (st) return st;
    *bytes = plan.total;
    return GDN_OK;
}

int gdn_chunk_fwd_launch_count(const gdn_fwd_args* args) {
    FwdPlan plan;
    return plan_fwd(args, &plan) ? -1 : plan.launches;
}

gdn_status gdn_chunk_fwd(const gdn_fwd_args* args, void* workspace, size_t workspace_bytes,
                         void* stream) {
    FwdPlan plan;
    gdn_status st = plan_fwd(args, &plan);
    if (st) return st;
    if ((st = check_fwd_pointers(args, plan.p))) return st;
    if ((st = check_workspace(workspace, workspace_bytes, plan.total))) return st;
    (void)cudaGetLastError();  // launches below report only their own errors
    cudaStream_t s = (cudaStream_t)stream;
    return plan.use_tc ? launch_fwd_tc(plan, (char*)workspace, s)
                       : launch_fwd_simt(plan, (char*)workspace, s);
}

gdn_status gdn_chunk_bwd_workspace_size(const gdn_bwd_args* args, size_t* bytes) {
    if (!bytes) return GDN_ERR_INVALID_ARG;
    BwdPlan plan;
    gdn_status st = plan_bwd(args, &plan);
    if (st) return st;
    *bytes = plan.total;
    return GDN_OK;
}

int gdn_chunk_bwd_launch_count(const gdn_bwd_args* args) {
    BwdPlan plan;
    return plan_bwd(args, &plan) ? -1 : plan.launches;
}

gdn_status gdn_chunk_bwd(const gdn_bwd_args* args, void* workspace, size_t workspace_bytes,
                         void* stream) {
    BwdPlan plan;
    gdn_status st = plan_bwd(args, &plan);
    if (st) return st;
    if ((st = check_bwd_pointers(args, plan.b.f))) return st;
    if ((st = check_workspace(workspace, workspace_bytes, plan.total))) return st;
    (void)cudaGetLastError();
    return plan.use_tc ? launch_bwd_tc(plan, (char*)workspace, (cudaStream_t)stream)
                       : launch_bwd_simt(plan, (char*)workspace, (cudaStream_t)stream);
}

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported configuration";
        case GDN_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case GDN_ERR_CUDA: return "CUDA launch or runtime error";
        case GDN_ERR_TIMEOUT: return "device wait timed out";
        case GDN_ERR_DEVICE: return "device-side consistency check failed";
        case GDN_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of gdn_chunk_fwd_noalloc";
        default: return "unknown status";
    }
}

}  // extern "C"
