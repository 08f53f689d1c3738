// KDA backward: gradients of the forward layer with respect to q, k, v, g,
// beta, gate and the initial state, given dL/dy and dL/d(final state).
//
// The pages give the forward only (Kimi K3 report explainer, affta.cn,
// section "第一关：KDA 解决算得动": forget, corrective write with an update
// strength, read, output gate).  The reverse recurrence is that forward
// differentiated step by step; per token t, going backwards, with S_{t-1} the
// state before the token, alpha = exp(g_t) and dS = dL/dS_t:
//   S' = Diag(alpha) S_{t-1};  a = S'^T k;  u = beta (v - a);  S_t = S' + k u^T
//   o = S_t^T (scale q);  do = gate (.) dy;  dgate = dy (.) o
//   dS += scale q do^T;   dq = scale S_t do
//   du = dS^T k;  dv = beta du;  dbeta = du . (v - a);  da = -beta du
//   dk = dS u + S' da;  dS' = dS + k da^T;  dg = rowsum(dS' (.) S')
//   dS <- Diag(alpha) dS'
//
// Layout of the work: the columns of the state are independent in every step
// except through the row sums (dq, dk, dg) and dbeta, so one CTA owns one
// (sequence, head, 32-column slice of dv) and adds its share of those sums
// into fp32 outputs with atomics; dv, dgate and the initial-state gradient are
// per column and stored directly.  Thread i (one per key channel) holds row i
// of the state slice and of dS in registers; sums over the key channels (a, o,
// du) are a warp reduce-scatter plus a shared-memory combine across warps.
//
// States going backwards: a forward sweep stores the state every kBlk tokens
// (checkpoints); the reverse sweep re-runs each block forwards from its
// checkpoint, keeping the block's states in per-CTA scratch, then walks the
// block backwards.  Every state row is written and read back by the thread
// that owns it.  fp32 throughout; the inputs are bf16 or fp32.
#include "kda.h"
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBlk = 64;   // tokens between checkpoints
constexpr int kCols = 32;  // state columns per CTA

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dy;
    const int32_t *cu;
    const float *s0, *dsT;
    float *dq, *dk, *dv, *dg, *dbeta, *dgate, *ds0;
    float *ckpt, *scratch;
    int N, H, DV, T;
    float scale;
};

// x[c] summed over the 32 lanes of the warp, for every c; lane c returns
// column c.  Recursive halving: at width s a lane keeps the half of its
// columns selected by bit s of its lane id and adds the partner's copy.
KDA_DEVICE float reduce_scatter32(float (&x)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool up = lane & s;
#pragma unroll
        for (int m = 0; m < s; ++m) {
            const float send = up ? x[m] : x[m + s];
            const float keep = up ? x[m + s] : x[m];
            x[m] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return x[0];
}

// Column sums over all key channels of the CTA: out[c] = sum_i x_i[c].
// Two barriers: the first also publishes the token's shared inputs.
template <int NW>
KDA_DEVICE void col_sum(float (&x)[32], float *red, float *out, int warp, int lane) {
    red[warp * 32 + lane] = reduce_scatter32(x, lane);
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) t += red[w * 32 + lane];
        out[lane] = t;
    }
    __syncthreads();
}

template <int DK, typename T>
__global__ void __launch_bounds__(DK) bwd_kernel(BwdParams p) {
    constexpr int NW = DK / 32;
    // per-token column data, double-buffered by token parity so that a fast
    // thread writing token t + 1 never overwrites what a slow one still reads
    __shared__ float red[NW * 32];
    __shared__ float cv[2][32], cgt[2][32], cdy[2][32];
    __shared__ float ca[2][32], co[2][32], cdu[2][32];

    const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
    const int nh = blockIdx.x, n = nh / p.H, h = nh % p.H;
    const int j0 = blockIdx.y * kCols;
    const int H = p.H, DV = p.DV;
    // offsets clamped into [0, T]: any offsets keep every access in bounds
    const int bos = min(max(p.cu[n], 0), p.T);
    const int eos = min(max(p.cu[n + 1], bos), p.T);
    const int L = eos - bos;
    const int nb = (L + kBlk - 1) / kBlk;
    const long ck0 = bos / kBlk + n;  // first checkpoint slot of the sequence
    const T *q = (const T *)p.q, *k = (const T *)p.k, *v = (const T *)p.v, *g = (const T *)p.g;
    const T *beta = (const T *)p.beta, *gate = (const T *)p.gate, *dy = (const T *)p.dy;
    const float scale = p.scale;
    float *scr = p.scratch + ((size_t)(nh * gridDim.y + blockIdx.y) * kBlk * DK + i) * kCols;
    auto ck_row = [&](int b) { return p.ckpt + (((size_t)(ck0 + b) * H + h) * DK + i) * DV + j0; };
    auto save = [](float *dst, const float (&x)[32]) {
#pragma unroll
        for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
    };
    auto load = [](const float *src, float (&x)[32]) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(src + c);
            x[c] = f.x; x[c + 1] = f.y; x[c + 2] = f.z; x[c + 3] = f.w;
        }
    };

    // S <- the state after token t (S holds the state before it)
    auto forward_token = [&](int t, float (&S)[32]) {
        const int par = t & 1;
        const size_t r = (size_t)t * H + h;
        const float ki = ld(k + r * DK + i);
        const float al = __expf(ld(g + r * DK + i));
        const float bt = ld(beta + r);
        if (i < 32) cv[par][i] = ld(v + r * DV + j0 + i);
        float x[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            S[c] *= al;
            x[c] = S[c] * ki;
        }
        col_sum<NW>(x, red, ca[par], warp, lane);
#pragma unroll
        for (int c = 0; c < 32; ++c) S[c] += ki * (bt * (cv[par][c] - ca[par][c]));
    };

    // ---- forward sweep: a checkpoint at the start of every block
    float S[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) S[c] = p.s0 ? p.s0[((size_t)nh * DK + i) * DV + j0 + c] : 0.f;
    for (int b = 0; b < nb; ++b) {
        save(ck_row(b), S);
        if (b + 1 < nb)
            for (int t = bos + b * kBlk; t < bos + (b + 1) * kBlk; ++t) forward_token(t, S);
    }

    // ---- reverse sweep
    float dS[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) dS[c] = p.dsT ? p.dsT[((size_t)nh * DK + i) * DV + j0 + c] : 0.f;
    for (int b = nb - 1; b >= 0; --b) {
        const int tb = bos + b * kBlk, te = min(eos, tb + kBlk);
        // the last token walked (tb + kBlk of the previous block, or the
        // forward sweep's) may share a buffer parity with the first one below
        __syncthreads();
        load(ck_row(b), S);
        for (int t = tb; t < te; ++t) {  // the block's states S_{t-1}, forwards
            save(scr + (size_t)(t - tb) * DK * kCols, S);
            if (t + 1 < te) forward_token(t, S);
        }
        for (int t = te - 1; t >= tb; --t) {
            const int par = t & 1;
            const size_t r = (size_t)t * H + h;
            const float ki = ld(k + r * DK + i), qi = ld(q + r * DK + i);
            const float al = __expf(ld(g + r * DK + i));
            const float bt = ld(beta + r);
            if (i < 32) {
                const size_t rc = r * DV + j0 + i;
                cv[par][i] = ld(v + rc);
                cgt[par][i] = gate ? ld(gate + rc) : 1.f;
                cdy[par][i] = ld(dy + rc);
            }
            float Sp[32], x[32];
            load(scr + (size_t)(t - tb) * DK * kCols, Sp);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                Sp[c] *= al;
                x[c] = Sp[c] * ki;
            }
            col_sum<NW>(x, red, ca[par], warp, lane);  // a = S'^T k
            // u_c = beta (v_c - a_c);  S_t = S' + k u^T;  o = S_t^T (scale q)
#pragma unroll
            for (int c = 0; c < 32; ++c)
                x[c] = (Sp[c] + ki * (bt * (cv[par][c] - ca[par][c]))) * (scale * qi);
            col_sum<NW>(x, red, co[par], warp, lane);
            if (i < 32 && p.dgate) p.dgate[r * DV + j0 + i] = cdy[par][i] * co[par][i];
            float dqi = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float doc = cgt[par][c] * cdy[par][c];
                const float st = Sp[c] + ki * (bt * (cv[par][c] - ca[par][c]));
                dqi += st * doc;
                dS[c] += scale * qi * doc;
                x[c] = dS[c] * ki;
            }
            col_sum<NW>(x, red, cdu[par], warp, lane);  // du = dS^T k
            if (i < 32) p.dv[r * DV + j0 + i] = bt * cdu[par][i];
            if (i == 0) {
                float db = 0.f;
#pragma unroll
                for (int c = 0; c < 32; ++c) db += cdu[par][c] * (cv[par][c] - ca[par][c]);
                atomicAdd(p.dbeta + r, db);
            }
            float dki = 0.f, dgi = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float uc = bt * (cv[par][c] - ca[par][c]);
                const float da = -bt * cdu[par][c];
                dki += dS[c] * uc + Sp[c] * da;
                const float dsp = dS[c] + ki * da;
                dgi += dsp * Sp[c];
                dS[c] = al * dsp;
            }
            atomicAdd(p.dq + r * DK + i, scale * dqi);
            atomicAdd(p.dk + r * DK + i, dki);
            atomicAdd(p.dg + r * DK + i, dgi);
        }
    }
    if (p.ds0) {
#pragma unroll
        for (int c = 0; c < 32; ++c) p.ds0[((size_t)nh * DK + i) * DV + j0 + c] = dS[c];
    }
}

template <int DK, typename T>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t st) {
    bwd_kernel<DK, T><<<dim3((unsigned)(p.N * p.H), (unsigned)(p.DV / kCols)), DK, 0, st>>>(p);
    return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t ckpt_bytes(long T, long N, long H, long dk, long dv) {
    return align256((size_t)(T / kBlk + N) * H * dk * dv * sizeof(float));
}

size_t scratch_bytes(long N, long H, long dk, long dv) {
    return align256((size_t)N * H * dv * kBlk * dk * sizeof(float));
}

bool ok_dim(int d) { return d == 64 || d == 128; }

}  // namespace
}  // namespace kda

extern "C" {

size_t kda_bwd_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                              int32_t dv) {
    if (total_tokens < 0 || num_seqs < 0 || H < 1 || !kda::ok_dim(dk) || !kda::ok_dim(dv)) return 0;
    return kda::ckpt_bytes(total_tokens, num_seqs, H, dk, dv) +
           kda::scratch_bytes(num_seqs, H, dk, dv);
}

int kda_bwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
            const void *gate, const void *dy, const int32_t *cu_seqlens,
            const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens, int32_t H,
            int32_t dk, int32_t dv, kda_dtype dtype, float scale, const float *initial_state,
            const float *d_final_state, float *dq, float *dk_out, float *dv_out, float *dg,
            float *dbeta, float *dgate, float *d_initial_state, void *workspace,
            size_t workspace_bytes, kda_stream_t stream) {
    if (num_seqs < 0 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!kda::ok_dim(dk) || !kda::ok_dim(dv)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (dgate && !gate) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_tokens)
            return KDA_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    }
    if (num_seqs == 0) return KDA_OK;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 &&
        (!q || !k || !v || !g || !beta || !dy || !dq || !dk_out || !dv_out || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const void *in[] = {q, k, v, g, beta, gate, dy};
    for (const void *ptr : in)
        if (ptr && (uintptr_t)ptr % esz) return KDA_ERR_ALIGNMENT;
    const void *out[] = {dq, dk_out, dv_out, dg, dbeta, dgate, d_initial_state, initial_state,
                         d_final_state};
    for (const void *ptr : out)
        if (ptr && (uintptr_t)ptr % 4) return KDA_ERR_ALIGNMENT;
    if ((long)num_seqs * H > 0x7fffffffL) return KDA_ERR_UNSUPPORTED;
    const size_t need = kda_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if ((uintptr_t)workspace % 256) return KDA_ERR_ALIGNMENT;

    cudaStream_t st = (cudaStream_t)stream;
    // the row sums and dbeta are accumulated across column slices
    const size_t tk = (size_t)total_tokens * H;
    if (tk > 0) {
        if (cudaMemsetAsync(dq, 0, tk * dk * sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(dk_out, 0, tk * dk * sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(dg, 0, tk * dk * sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(dbeta, 0, tk * sizeof(float), st) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    kda::BwdParams p{};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.gate = gate; p.dy = dy;
    p.cu = cu_seqlens;
    p.s0 = initial_state; p.dsT = d_final_state;
    p.dq = dq; p.dk = dk_out; p.dv = dv_out; p.dg = dg; p.dbeta = dbeta; p.dgate = dgate;
    p.ds0 = d_initial_state;
    p.ckpt = (float *)workspace;
    p.scratch = (float *)((char *)workspace + kda::ckpt_bytes(total_tokens, num_seqs, H, dk, dv));
    p.N = num_seqs; p.H = H; p.DV = dv; p.T = total_tokens;
    p.scale = scale;
    cudaError_t e;
    const bool bf = dtype == KDA_DTYPE_BF16;
    if (dk == 128)
        e = bf ? kda::launch_bwd_t<128, __nv_bfloat16>(p, st) : kda::launch_bwd_t<128, float>(p, st);
    else
        e = bf ? kda::launch_bwd_t<64, __nv_bfloat16>(p, st) : kda::launch_bwd_t<64, float>(p, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
