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
// (sequence, head, 8-column slice of dv) and adds its share of those sums
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

constexpr int kBlk = 16;   // tokens between checkpoints (a block's states stay L2-resident)
constexpr int kAhead = 8;  // tokens ahead whose lines are prefetched into L2
constexpr int kCols = 8;   // state columns per CTA (NC below)
constexpr int NC = kCols;

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dy;
    const int32_t *cu;
    const float *s0, *dsT;
    float *dq, *dk, *dv, *dg, *dbeta, *dgate, *ds0;
    float *ckpt, *scratch;
    int N, H, DV, T;
    float scale;
};

// x[c] (c < NC) summed over the 32 lanes of the warp; lane l returns column
// l % NC.  With NC < 32 the lanes 16 (and 8) apart are added first.  Then
// recursive halving: at width s a lane keeps the half of its columns selected
// by bit s of its lane id and adds the partner's copy of that half.
KDA_DEVICE float reduce_scatter(float (&x)[NC], int lane) {
    static_assert(NC == 8 || NC == 16 || NC == 32, "slice width");
    if constexpr (NC <= 16) {
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] += __shfl_xor_sync(0xffffffffu, x[c], 16);
    }
    if constexpr (NC <= 8) {
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] += __shfl_xor_sync(0xffffffffu, x[c], 8);
    }
#pragma unroll
    for (int s = NC / 2; s >= 1; s >>= 1) {
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
KDA_DEVICE void col_sum(float (&x)[NC], float *red, float *out, int warp, int lane) {
    const float sx = reduce_scatter(x, lane);
    if (lane < NC) red[warp * NC + lane] = sx;
    __syncthreads();
    if (warp == 0 && lane < NC) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) t += red[w * NC + lane];
        out[lane] = t;
    }
    __syncthreads();
}

// Three column sums and one scalar sum in one exchange: out[0, NC) = sum x,
// out[NC, 2 NC) = sum y, out[2 NC, 3 NC) = sum z, out[3 NC] = sum w.
constexpr int kRed3 = 3 * NC + 1;
template <int NW>
KDA_DEVICE void col_sum3(float (&x)[NC], float (&y)[NC], float (&z)[NC], float w, float *red,
                         float *out, int warp, int lane) {
    const float sx = reduce_scatter(x, lane);
    const float sy = reduce_scatter(y, lane);
    const float sz = reduce_scatter(z, lane);
    const float sw = warp_sum(w);
    float *r = red + warp * kRed3;
    if (lane < NC) {
        r[lane] = sx;
        r[NC + lane] = sy;
        r[2 * NC + lane] = sz;
    }
    if (lane == 0) r[3 * NC] = sw;
    __syncthreads();
    for (int e = threadIdx.x; e < kRed3; e += 32 * NW) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < NW; ++q) t += red[q * kRed3 + e];
        out[e] = t;
    }
    __syncthreads();
}

KDA_DEVICE void prefetch_l2(const void *ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

struct FwdIn {  // one token's inputs to the forward step (v: column i, i < NC)
    float k, g, beta, v;
};
struct RevIn {  // one token's inputs to the reverse step (v, gate, dy: column i, i < NC)
    float k, q, g, beta, v, gate, dy;
};

template <int DK, typename T>
// 512 threads per SM at least (four 128-thread CTAs): more chains share each SM
__global__ void __launch_bounds__(DK, 512 / DK) bwd_kernel(BwdParams p) {
    constexpr int NW = DK / 32;
    // per-token shared data, double-buffered by token parity so that a fast
    // thread writing the next token never overwrites what a slow one still
    // reads (the barriers of one token separate uses two tokens apart)
    __shared__ float red[NW * kRed3];
    __shared__ float cv[2][NC], cgt[2][NC], cdy[2][NC];
    __shared__ float ca[2][NC], cs[2][kRed3];

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
    auto save = [](float *dst, const float (&x)[NC]) {
#pragma unroll
        for (int c = 0; c < NC; c += 4)
            *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
    };
    auto load = [](const float *src, float (&x)[NC]) {
#pragma unroll
        for (int c = 0; c < NC; c += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(src + c);
            x[c] = f.x; x[c + 1] = f.y; x[c + 2] = f.z; x[c + 3] = f.w;
        }
    };
    auto load_fwd = [&](int t) {
        const size_t r = (size_t)t * H + h;
        FwdIn x;
        x.k = ld(k + r * DK + i);
        x.g = ld(g + r * DK + i);
        x.beta = ld(beta + r);
        x.v = i < NC ? ld(v + r * DV + j0 + i) : 0.f;
        return x;
    };
    auto load_rev = [&](int t) {
        const size_t r = (size_t)t * H + h;
        RevIn x;
        x.k = ld(k + r * DK + i);
        x.q = ld(q + r * DK + i);
        x.g = ld(g + r * DK + i);
        x.beta = ld(beta + r);
        x.v = x.gate = x.dy = 0.f;
        if (i < NC) {
            const size_t rc = r * DV + j0 + i;
            x.v = ld(v + rc);
            x.gate = gate ? ld(gate + rc) : 1.f;
            x.dy = ld(dy + rc);
        }
        return x;
    };

    // L2 prefetch of token t's input lines (one thread per 128-byte line of a
    // row; t must be a token of this sequence)
    constexpr int kLine = 128 / (int)sizeof(T);
    auto prefetch_in = [&](int t, bool rev) {
        const size_t r = (size_t)t * H + h;
        if (i % kLine == 0) {
            prefetch_l2(k + r * DK + i);
            prefetch_l2(g + r * DK + i);
            if (rev) prefetch_l2(q + r * DK + i);
        }
        if (i == 0) {
            prefetch_l2(beta + r);
            prefetch_l2(v + r * DV + j0);
            if (rev) {
                prefetch_l2(dy + r * DV + j0);
                if (gate) prefetch_l2(gate + r * DV + j0);
            }
        }
    };

    // S <- the state after token t (S holds the state before it)
    auto fwd_step = [&](int t, const FwdIn &in, float (&S)[NC]) {
        const int par = t & 1;
        const float al = __expf(in.g);
        if (i < NC) cv[par][i] = in.v;
        float x[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            S[c] *= al;
            x[c] = S[c] * in.k;
        }
        col_sum<NW>(x, red, ca[par], warp, lane);
#pragma unroll
        for (int c = 0; c < NC; ++c) S[c] += in.k * (in.beta * (cv[par][c] - ca[par][c]));
    };
    // forward over tokens [t0, t1) with the next token's inputs in flight
    auto fwd_run = [&](int t0, int t1, float (&S)[NC], bool keep) {
        if (t0 >= t1) return;
        FwdIn cur = load_fwd(t0);
        for (int t = t0; t < t0 + kAhead && t < t1; ++t) prefetch_in(t, false);
        for (int t = t0; t < t1; ++t) {
            if (t + kAhead < t1) prefetch_in(t + kAhead, false);
            if (keep) save(scr + (size_t)(t - t0) * DK * kCols, S);
            else if ((t - bos) % kBlk == 0) save(ck_row((t - bos) / kBlk), S);
            const FwdIn nxt = t + 1 < t1 ? load_fwd(t + 1) : cur;
            fwd_step(t, cur, S);
            cur = nxt;
        }
    };

    // ---- forward sweep: a checkpoint at the start of every block
    float S[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) S[c] = p.s0 ? p.s0[((size_t)nh * DK + i) * DV + j0 + c] : 0.f;
    if (nb > 0) {
        fwd_run(bos, bos + (nb - 1) * kBlk, S, false);
        save(ck_row(nb - 1), S);
    }

    // ---- reverse sweep
    float dS[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) dS[c] = p.dsT ? p.dsT[((size_t)nh * DK + i) * DV + j0 + c] : 0.f;
    for (int b = nb - 1; b >= 0; --b) {
        const int tb = bos + b * kBlk, te = min(eos, tb + kBlk);
        // the last token walked (tb + kBlk of the previous block, or the
        // forward sweep's) may share a buffer parity with the first one below
        __syncthreads();
        load(ck_row(b), S);
        // the block's states S_{t-1} into scratch (the last one saved, not stepped)
        fwd_run(tb, te - 1, S, true);
        save(scr + (size_t)(te - 1 - tb) * DK * kCols, S);

        RevIn cur = load_rev(te - 1);
        float Sp[NC];
        load(scr + (size_t)(te - 1 - tb) * DK * kCols, Sp);
        for (int t = te - 1; t >= tb && t >= te - kAhead; --t) {
            prefetch_in(t, true);
            prefetch_l2(scr + (size_t)(t - tb) * DK * kCols);
        }
        for (int t = te - 1; t >= tb; --t) {
            const int par = t & 1;
            const size_t r = (size_t)t * H + h;
            if (t - kAhead >= tb) {
                prefetch_in(t - kAhead, true);
                prefetch_l2(scr + (size_t)(t - kAhead - tb) * DK * kCols);
            }
            RevIn nxt = cur;
            float Sn[NC];
            if (t > tb) {
                nxt = load_rev(t - 1);
                load(scr + (size_t)(t - 1 - tb) * DK * kCols, Sn);
            }
            const float al = __expf(cur.g);
            if (i < NC) {
                cv[par][i] = cur.v;
                cgt[par][i] = cur.gate;
                cdy[par][i] = cur.dy;
            }
            // one exchange: a = S'^T k, b = S'^T q, c = dS^T k (dS = dL/dS_t
            // without this token's read) and k.q
            float x[NC], y[NC], z[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                Sp[c] *= al;
                x[c] = Sp[c] * cur.k;
                y[c] = Sp[c] * cur.q;
                z[c] = dS[c] * cur.k;
            }
            col_sum3<NW>(x, y, z, cur.k * cur.q, red, cs[par], warp, lane);
            const float *A = cs[par], *Bq = cs[par] + NC, *C = cs[par] + 2 * NC;
            const float kq = cs[par][3 * NC], bt = cur.beta;
            if (i < NC) {  // per column: u, o (= scale (b + (k.q) u)), du, dv, dgate
                const float u = bt * (cur.v - A[i]);
                const float o = scale * (Bq[i] + kq * u);
                const float du = C[i] + scale * kq * (cur.gate * cur.dy);
                p.dv[r * DV + j0 + i] = bt * du;
                if (p.dgate) p.dgate[r * DV + j0 + i] = cur.dy * o;
            }
            if (i == 0) {
                float db = 0.f;
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const float du = C[c] + scale * kq * (cgt[par][c] * cdy[par][c]);
                    db += du * (cv[par][c] - A[c]);
                }
                atomicAdd(p.dbeta + r, db);
            }
            float dqi = 0.f, dki = 0.f, dgi = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const float doc = cgt[par][c] * cdy[par][c];
                const float uc = bt * (cv[par][c] - A[c]);
                dqi += (Sp[c] + cur.k * uc) * doc;              // S_t do
                const float dsc = dS[c] + scale * cur.q * doc;  // dL/dS_t
                const float da = -bt * (C[c] + scale * kq * doc);
                dki += dsc * uc + Sp[c] * da;
                const float dsp = dsc + cur.k * da;              // dL/dS'
                dgi += dsp * Sp[c];
                dS[c] = al * dsp;                                // dL/dS_{t-1}
            }
            atomicAdd(p.dq + r * DK + i, scale * dqi);
            atomicAdd(p.dk + r * DK + i, dki);
            atomicAdd(p.dg + r * DK + i, dgi);
            cur = nxt;
#pragma unroll
            for (int c = 0; c < NC; ++c) Sp[c] = Sn[c];
        }
    }
    if (p.ds0) {
#pragma unroll
        for (int c = 0; c < NC; ++c) p.ds0[((size_t)nh * DK + i) * DV + j0 + c] = dS[c];
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
