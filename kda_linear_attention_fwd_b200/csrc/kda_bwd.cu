// KDA backward: gradients of the forward layer with respect to q, k, v, g,
// beta, gate and the initial state, given dL/dy and dL/d(final state).
//
// The pages give the forward only (Kimi K3 report explainer, affta.cn,
// section "第一关：KDA 解决算得动": forget, corrective write with an update
// strength, read, output gate).  This is its 16-token chunk form
// (prism.simon-ai.net, section "计算范式演进：从递归低效到 GPU 友好的 Chunk
// Recurrent"; the decay as a transform inside a 16-token tile, section
// "数值稳定性与 Co-Design：BF16 约束下的衰减控制策略") differentiated by the
// chain rule.  Per chunk of C = 16 rows (rows past a sequence's end are zero,
// with g = 0), G = the inclusive running sum of g over the chunk's rows,
// E = exp(G), s = scale, S = the state entering the chunk:
//   Kd = K (.) E,  Ki = K (.) E^-1,  Qd = s Q (.) E,  Kb = K (.) exp(G_C - G)
//   A = strict_tril(Kd Ki^T),  P = tril(Qd Ki^T),  X = (I + Diag(beta) A)^-1
//   T = X Diag(beta),  W = T Kd,  U0 = T V
//   U = U0 - W S,  O = Qd S + P U,  y = gate (.) O
//   S' = Diag(gamma_C) S + Kb^T U        (G_C = G of the last row, gamma_C = exp(G_C))
// Going backwards, with dS' = dL/dS' and dO = gate (.) dy:
//   dU = P^T dO + Kb dS',   dS = Qd^T dO + Diag(gamma_C) dS' - W^T dU    (the chain)
//   dQd = dO S^T,  dW = -dU S^T,  dKb = U dS'^T,  dgamma_C = rowsum(dS' (.) S)
//   dP = tril(dO U^T),  dT = dU V^T + dW Kd^T,  dV = T^T dU,  dKd = T^T dW
//   M = X^T dT Diag(beta),  dL = -M X^T
//   dbeta = colsum(X (.) dT) + rowsum(strict(dL) (.) A),  dA = Diag(beta) strict(dL)
//   dKd += dA Ki,  dKi = dA^T Kd + dP^T Qd,  dQd += dP Ki
//   dK = dKd (.) E + dKi (.) E^-1 + dKb (.) exp(G_C - G),  dQ = s dQd (.) E
//   dG = dKd (.) Kd - dKi (.) Ki + dQd (.) Qd - dKb (.) Kb; the last row adds
//        colsum(dKb (.) Kb) + dgamma_C (.) gamma_C;  dg = suffix sums of dG over the rows
//
// Three launches, all fp32 arithmetic on bf16 or fp32 inputs:
//   prep_kernel   per (chunk, head), parallel: W, Qd, Kb, U0, P, gamma_C -> workspace
//   chain_kernel  two independent sequential passes side by side:
//     fwd_chain   per (sequence, head, 32 state columns), chunks in order: the
//                 state entering each chunk and U -> workspace; dgate = dy (.) O
//     rev_chain   per (sequence, head, 32 columns), chunks in reverse: dS' and
//                 dU -> workspace; dL/d(initial state)
//   grad_kernel   per (chunk, head), parallel: the other gradients from the
//                 chunk's inputs, S, dS', U and dU; its three products with a
//                 whole state run on split-tf32 tensor-core tiles
// Every output element is written by exactly one thread (no atomics), so the
// results do not depend on scheduling.
#include "kda.h"
#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using sm100::cp_async16;
using sm100::cp_async_commit;
using sm100::cp_async_wait;

constexpr int C = 16;          // tokens per chunk
constexpr int kThreads = 256;  // prep and grad CTAs, and each half of a chain CTA
constexpr int kWarps = kThreads / 32;
constexpr int NC = 16;         // state columns of one half of a chain CTA
constexpr int kHalves = 2;     // chain CTAs: two halves of 256 threads share the chunk operands
constexpr int kChainThreads = kHalves * kThreads;

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dy;
    const int32_t *cu;
    const float *s0, *dsT;
    float *dq, *dk, *dv, *dg, *dbeta, *dgate, *ds0;
    float *prep;  // per (slot, head): the prep block (Blk below)
    float *Sst;   // per (slot, head): the state entering the chunk, [DK][DV]
    float *dSst;  // per (slot, head): dL/d(state leaving the chunk), [DK][DV]
    float *Ust;   // per (slot, head): U, [C][DV]
    float *dUst;  // per (slot, head): dL/dU, [C][DV]
    int N, H, T;
    float scale;
};

// Offsets (floats) inside one prep block: W, Qd, Kb [C][DK], U0 [C][DV],
// P [C][C], gamma_C [DK].  Every offset and the block size are
// multiples of four floats (dk, dv in {64, 128}), so 16-byte copies stay
// aligned.
template <int DK, int DV> struct Blk {
    static constexpr int W = 0, QD = C * DK, KB = 2 * C * DK, U0 = 3 * C * DK;
    static constexpr int P = U0 + C * DV, GC = P + C * C, size = GC + DK;
};

// Chunk slots: chunk c of sequence n is slot cu[n] / C + n + c.  A sequence of
// L tokens has ceil(L / C) chunks, and the slots of different sequences do
// not overlap; all fit below total_tokens / C + num_seqs.
struct Seq {
    int bos, len, nb;
    long slot0;
};

KDA_DEVICE int clamp_off(const BwdParams &p, int n) { return min(max(p.cu[n], 0), p.T); }

KDA_DEVICE Seq seq_of(const BwdParams &p, int n) {
    Seq s;
    s.bos = clamp_off(p, n);
    const int eos = min(max(p.cu[n + 1], s.bos), p.T);
    s.len = eos - s.bos;
    s.nb = (s.len + C - 1) / C;
    s.slot0 = s.bos / C + n;
    return s;
}

// The sequence and chunk of a slot (false: no chunk uses it).  Offsets are
// clamped as in seq_of, so any offsets keep every access in bounds.
KDA_DEVICE bool chunk_of_slot(const BwdParams &p, long slot, Seq &s, int &c) {
    int lo = 0, hi = p.N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long)(clamp_off(p, mid) / C) + mid <= slot) lo = mid;
        else hi = mid - 1;
    }
    s = seq_of(p, lo);
    const long cc = slot - s.slot0;
    if (cc < 0 || cc >= s.nb) return false;
    c = (int)cc;
    return true;
}

KDA_DEVICE float dot4(float4 a, float4 b, float acc) {
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    return fmaf(a.w, b.w, acc);
}

// ---- the chunk's operands in shared memory (prep_kernel and grad_kernel)
template <int DK, int DV> struct alignas(16) PrepSm {
    static constexpr int LK = DK + 4;                        // padded row strides (floats)
    static constexpr int LM = (DK > DV ? DK : DV) + 4;
    float kd[C][LK], ki[C][LK], qd[C][LK], kb[C][LK], gs[C][LK];  // gs: G
    float vs[C][LM];                                         // V (grad_kernel: then dKd)
    float A[C][C + 1], P[C][C + 1], X[C][C + 1], Tm[C][C + 1];
    float beta[C];
    float gc[DK];                                            // gamma_C
};

// Loads the chunk (rows t0 .. t0 + n - 1 of head h; the rest zero) and forms
// G, Kd, Ki, Qd, Kb, gamma_C, A, P, X and T in shared memory.
template <int DK, int DV, typename T>
KDA_DEVICE void prep_chunk(const BwdParams &p, PrepSm<DK, DV> &sm, int h, int t0, int n) {
    const int tid = threadIdx.x, H = p.H;
    const T *q = (const T *)p.q, *k = (const T *)p.k, *g = (const T *)p.g;
    const T *v = (const T *)p.v, *beta = (const T *)p.beta;
    // all of a thread's loads are issued before its first shared-memory store
    constexpr int NK = C * DK / kThreads, NV = C * DV / kThreads;
    static_assert(NK * kThreads == C * DK && NV * kThreads == C * DV, "whole rows per pass");
    float kv[NK], qv[NK], gv[NK], vv[NV];
#pragma unroll
    for (int u = 0; u < NK; ++u) {
        const int e = tid + u * kThreads, r = e / DK, i = e % DK;
        kv[u] = qv[u] = gv[u] = 0.f;
        if (r < n) {
            const size_t o = ((size_t)(t0 + r) * H + h) * DK + i;
            kv[u] = ld(k + o);
            qv[u] = ld(q + o);
            gv[u] = ld(g + o);
        }
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int e = tid + u * kThreads, r = e / DV, j = e % DV;
        vv[u] = r < n ? ld(v + ((size_t)(t0 + r) * H + h) * DV + j) : 0.f;
    }
    const float bv = tid < n ? ld(beta + (size_t)(t0 + tid) * H + h) : 0.f;
#pragma unroll
    for (int u = 0; u < NK; ++u) {
        const int e = tid + u * kThreads, r = e / DK, i = e % DK;
        sm.kd[r][i] = kv[u];
        sm.qd[r][i] = qv[u];
        sm.gs[r][i] = gv[u];
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int e = tid + u * kThreads;
        sm.vs[e / DV][e % DV] = vv[u];
    }
    if (tid < C) sm.beta[tid] = bv;
    __syncthreads();
    if (tid < DK) {  // decay: one thread per key channel, down the rows
        const int i = tid;
        float G = 0.f;
#pragma unroll
        for (int r = 0; r < C; ++r) {
            G += sm.gs[r][i];
            sm.gs[r][i] = G;
        }
        const float GC = G;
        sm.gc[i] = expf(GC);
#pragma unroll 4
        for (int r = 0; r < C; ++r) {
            const float Gr = sm.gs[r][i], kv = sm.kd[r][i];
            const float e = expf(Gr);
            sm.kd[r][i] = kv * e;
            sm.ki[r][i] = kv * expf(-Gr);
            sm.qd[r][i] = p.scale * sm.qd[r][i] * e;
            sm.kb[r][i] = kv * expf(GC - Gr);
        }
    }
    __syncthreads();
    {  // A and P: thread (r, s)
        const int r = tid >> 4, s = tid & 15;
        const float4 *kd4 = reinterpret_cast<const float4 *>(sm.kd[r]);
        const float4 *qd4 = reinterpret_cast<const float4 *>(sm.qd[r]);
        const float4 *ki4 = reinterpret_cast<const float4 *>(sm.ki[s]);
        float a = 0.f, pp = 0.f;
#pragma unroll 8
        for (int c4 = 0; c4 < DK / 4; ++c4) {
            const float4 x = ki4[c4];
            a = dot4(kd4[c4], x, a);
            pp = dot4(qd4[c4], x, pp);
        }
        sm.A[r][s] = r > s ? a : 0.f;
        sm.P[r][s] = r >= s ? pp : 0.f;
    }
    __syncthreads();
    if (tid < C) {  // X = (I + Diag(beta) A)^-1 by forward substitution, column s per lane
        const int s = tid;
        float x[C];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) acc = fmaf(sm.A[r][m], x[m], acc);
            x[r] = r < s ? 0.f : (r == s ? 1.f : -sm.beta[r] * acc);
        }
        const float bs = sm.beta[s];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            sm.X[r][s] = x[r];
            sm.Tm[r][s] = x[r] * bs;
        }
    }
    __syncthreads();
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kThreads) prep_kernel(BwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<PrepSm<DK, DV> *>(smem_raw);
    using B = Blk<DK, DV>;
    const long slot = blockIdx.x;
    const int h = blockIdx.y, tid = threadIdx.x;
    Seq s;
    int c;
    if (!chunk_of_slot(p, slot, s, c)) return;
    prep_chunk<DK, DV, T>(p, sm, h, s.bos + c * C, min(C, s.len - c * C));
    float *out = p.prep + ((size_t)slot * p.H + h) * B::size;
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, i = e % DK;
        float w = 0.f;
#pragma unroll
        for (int m = 0; m < C; ++m) w = fmaf(sm.Tm[r][m], sm.kd[m][i], w);  // T is lower triangular
        out[B::W + e] = w;
        out[B::QD + e] = sm.qd[r][i];
        out[B::KB + e] = sm.kb[r][i];
    }
    for (int e = tid; e < C * DV; e += kThreads) {
        const int r = e / DV, j = e % DV;
        float u = 0.f;
#pragma unroll
        for (int m = 0; m < C; ++m) u = fmaf(sm.Tm[r][m], sm.vs[m][j], u);
        out[B::U0 + e] = u;
    }
    out[B::P + tid] = sm.P[tid >> 4][tid & 15];
    for (int i = tid; i < DK; i += kThreads) out[B::GC + i] = sm.gc[i];
}

// ---- split-tf32 tensor-core tiles (mma.sync m16n8k8) for the products of
// grad_kernel that run over a whole state: fp32 accuracy from tf32 tiles by
// splitting each operand as x = hi + lo and forming hi*hi + hi*lo + lo*hi
// with fp32 accumulation (what is dropped is below 2^-20 relative).

// x = hi + lo: hi = x with the 13 low mantissa bits cleared (a tf32 value), lo
// = the exact remainder, of which the tensor core reads the tf32 part
// (|lo| < 2^-10 |x|, so the representation error is below 2^-20 |x|)
KDA_DEVICE void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}

KDA_DEVICE void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += A B for A = ah + al and B = (b0, b1) split here
KDA_DEVICE void mma3(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], float b0, float b1) {
    uint32_t bh0, bl0, bh1, bl1;
    split_tf32(b0, bh0, bl0);
    split_tf32(b1, bh1, bl1);
    mma_tf32(d, al, bh0, bh1);
    mma_tf32(d, ah, bl0, bl1);
    mma_tf32(d, ah, bh0, bh1);
}

// ---- the sequential passes: one CTA per (sequence, head, 2 NC state
// columns), two halves of 256 threads with NC columns each that share one copy
// of the chunk operands.  In a half, thread t owns column j = t % 16 and rows
// rg R .. rg R + R - 1 (rg = t / 16, R = DK / 16) of the state (or of its
// gradient) in registers; for the chunk's [C][NC] outputs it is thread (r, j)
// with r = rg.  Sums over the key channels: the two row groups of a warp are
// added with one shuffle, then the eight warps of the half through shared
// memory.
template <int DK> struct alignas(16) ChainSm {
    struct Buf {                   // one chunk's prep block (the rows this CTA needs)
        float wqk[3 * C * DK];     // W, Qd, Kb: [C][DK] each
        float pg[C * C + DK];      // P [C][C], gamma_C [DK]
        float u0[C * kHalves * NC];  // forward pass: U0 columns of this CTA, [C][2 NC]
        KDA_DEVICE const float *w() const { return wqk; }
        KDA_DEVICE const float *qd() const { return wqk + C * DK; }
        KDA_DEVICE const float *kb() const { return wqk + 2 * C * DK; }
        KDA_DEVICE const float *pm() const { return pg; }
        KDA_DEVICE const float *gc() const { return pg + C * C; }
    } buf[2];
    float red[kHalves][kWarps][C][32];  // partial sums per warp
    float xs[kHalves][2][C][NC];        // reverse pass: dO of the chunk (by iteration parity)
    float us[kHalves][C][NC];           // U (forward) or dU (reverse) of the chunk
};

// cp.async of chunk prep block `blk` into `b` (one group).
template <int DK, int DV>
KDA_DEVICE void fetch_prep(typename ChainSm<DK>::Buf &b, const float *blk, int j0, bool with_u0) {
    using B = Blk<DK, DV>;
    constexpr int NW = kHalves * NC;  // columns of the CTA
    const int tid = threadIdx.x;
    for (int e = tid; e < 3 * C * DK / 4; e += kChainThreads) cp_async16(b.wqk + 4 * e, blk + B::W + 4 * e, true);
    for (int e = tid; e < (C * C + DK) / 4; e += kChainThreads) cp_async16(b.pg + 4 * e, blk + B::P + 4 * e, true);
    if (with_u0 && tid < C * NW / 4) {
        const int r = tid / (NW / 4), c4 = tid % (NW / 4);
        cp_async16(b.u0 + r * NW + 4 * c4, blk + B::U0 + r * DV + j0 + 4 * c4, true);
    }
    cp_async_commit();
}

// x[0..R) . row segment (R consecutive floats of shared memory, 16-byte aligned)
template <int R> KDA_DEVICE float dot_rows(const float *seg, const float (&x)[R]) {
    float a = 0.f;
#pragma unroll
    for (int m4 = 0; m4 < R / 4; ++m4) {
        const float4 w = *reinterpret_cast<const float4 *>(seg + 4 * m4);
        a = fmaf(w.x, x[4 * m4], a);
        a = fmaf(w.y, x[4 * m4 + 1], a);
        a = fmaf(w.z, x[4 * m4 + 2], a);
        a = fmaf(w.w, x[4 * m4 + 3], a);
    }
    return a;
}

// x[0..R) += c * row segment
template <int R> KDA_DEVICE void axpy_rows(const float *seg, float c, float (&x)[R]) {
#pragma unroll
    for (int m4 = 0; m4 < R / 4; ++m4) {
        const float4 w = *reinterpret_cast<const float4 *>(seg + 4 * m4);
        x[4 * m4] = fmaf(w.x, c, x[4 * m4]);
        x[4 * m4 + 1] = fmaf(w.y, c, x[4 * m4 + 1]);
        x[4 * m4 + 2] = fmaf(w.z, c, x[4 * m4 + 2]);
        x[4 * m4 + 3] = fmaf(w.w, c, x[4 * m4 + 3]);
    }
}

// Forward pass over the chunks of one sequence: stores the state entering
// each chunk and U; dgate = dy (.) O.
template <int DK, int DV, typename T>
KDA_DEVICE void fwd_chain(const BwdParams &p, ChainSm<DK> &sm) {
    constexpr int R = DK / 16;
    using B = Blk<DK, DV>;
    const int hv = threadIdx.x / kThreads, tid = threadIdx.x % kThreads, lane = tid & 31, warp = tid >> 5;
    const int j = tid & 15, rg = tid >> 4, i0 = rg * R;
    const int nh = blockIdx.x, n = nh / p.H, h = nh % p.H, H = p.H;
    const int jc = blockIdx.y * kHalves * NC, j0 = jc + hv * NC;  // the CTA's and the half's first column
    auto &red = sm.red[hv];
    auto &us = sm.us[hv];
    const Seq s = seq_of(p, n);
    const T *dy = (const T *)p.dy;
    float S[R];
#pragma unroll
    for (int m = 0; m < R; ++m) S[m] = p.s0 ? p.s0[((size_t)nh * DK + i0 + m) * DV + j0 + j] : 0.f;
    if (s.nb == 0) return;
    auto blk = [&](int c) { return p.prep + ((size_t)(s.slot0 + c) * H + h) * B::size; };
    auto load_dy = [&](int c) {
        const int r = c * C + rg;
        return (p.dgate && r < s.len) ? ld(dy + ((size_t)(s.bos + r) * H + h) * DV + j0 + j) : 0.f;
    };
    fetch_prep<DK, DV>(sm.buf[0], blk(0), jc, true);
    float dyv = load_dy(0);
    for (int c = 0; c < s.nb; ++c) {
        const auto &b = sm.buf[c & 1];
        cp_async_wait<0>();
        __syncthreads();
        if (c + 1 < s.nb) fetch_prep<DK, DV>(sm.buf[(c + 1) & 1], blk(c + 1), jc, true);
        const size_t idx = (size_t)(s.slot0 + c) * H + h;
        float *Sg = p.Sst + idx * DK * DV + (size_t)i0 * DV + j0 + j;
#pragma unroll
        for (int m = 0; m < R; ++m) Sg[(size_t)m * DV] = S[m];
        // rows of W S and Qd S over this thread's key channels; lanes 0-15
        // keep the U sums of the warp's two row groups, lanes 16-31 the Qd S sums
        const bool hi = lane >= 16;
#pragma unroll
        for (int r = 0; r < C; ++r) {
            const float pu = dot_rows<R>(b.w() + r * DK + i0, S);
            const float pq = dot_rows<R>(b.qd() + r * DK + i0, S);
            const float send = hi ? pu : pq, keep = hi ? pq : pu;
            red[warp][r][lane] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        __syncthreads();
        float u = 0.f, qs = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            u += red[w][rg][j];
            qs += red[w][rg][16 + j];
        }
        u = b.u0[rg * kHalves * NC + hv * NC + j] - u;
        us[rg][j] = u;
        p.Ust[idx * C * DV + (size_t)rg * DV + j0 + j] = u;
        __syncthreads();
        float o = qs;  // O = Qd S + P U (P is zero above the diagonal)
#pragma unroll
        for (int r2 = 0; r2 < C; ++r2) o = fmaf(b.pm()[rg * C + r2], us[r2][j], o);
        if (p.dgate && c * C + rg < s.len)
            p.dgate[((size_t)(s.bos + c * C + rg) * H + h) * DV + j0 + j] = dyv * o;
        if (c + 1 < s.nb) dyv = load_dy(c + 1);
        // S <- Diag(gamma_C) S + Kb^T U
        const float *gc = b.gc() + i0;
#pragma unroll
        for (int m = 0; m < R; ++m) S[m] *= gc[m];
#pragma unroll
        for (int r = 0; r < C; ++r) axpy_rows<R>(b.kb() + r * DK + i0, us[r][j], S);
    }
}

// Reverse pass over the chunks of one sequence: stores dL/d(state leaving
// each chunk) and dU; writes dL/d(initial state).
template <int DK, int DV, typename T>
KDA_DEVICE void rev_chain(const BwdParams &p, ChainSm<DK> &sm) {
    constexpr int R = DK / 16;
    using B = Blk<DK, DV>;
    const int hv = threadIdx.x / kThreads, tid = threadIdx.x % kThreads, lane = tid & 31, warp = tid >> 5;
    const int j = tid & 15, rg = tid >> 4, i0 = rg * R;
    const int nh = blockIdx.x, n = nh / p.H, h = nh % p.H, H = p.H;
    const int jc = blockIdx.y * kHalves * NC, j0 = jc + hv * NC;  // the CTA's and the half's first column
    auto &red = sm.red[hv];
    auto &us = sm.us[hv];
    const Seq s = seq_of(p, n);
    const T *dy = (const T *)p.dy, *gate = (const T *)p.gate;
    float dS[R];
#pragma unroll
    for (int m = 0; m < R; ++m) dS[m] = p.dsT ? p.dsT[((size_t)nh * DK + i0 + m) * DV + j0 + j] : 0.f;
    auto blk = [&](int c) { return p.prep + ((size_t)(s.slot0 + c) * H + h) * B::size; };
    auto load_do = [&](int c) {
        const int r = c * C + rg;
        if (r >= s.len) return 0.f;
        const size_t o = ((size_t)(s.bos + r) * H + h) * DV + j0 + j;
        const float d = ld(dy + o);
        return gate ? ld(gate + o) * d : d;
    };
    auto &xs = sm.xs[hv];
    if (s.nb > 0) fetch_prep<DK, DV>(sm.buf[0], blk(s.nb - 1), jc, false);
    float dov = s.nb > 0 ? load_do(s.nb - 1) : 0.f;
    for (int it = 0; it < s.nb; ++it) {
        const int c = s.nb - 1 - it;
        const auto &b = sm.buf[it & 1];
        cp_async_wait<0>();
        __syncthreads();
        if (c > 0) fetch_prep<DK, DV>(sm.buf[(it + 1) & 1], blk(c - 1), jc, false);
        xs[it & 1][rg][j] = dov;
        const size_t idx = (size_t)(s.slot0 + c) * H + h;
        float *dSg = p.dSst + idx * DK * DV + (size_t)i0 * DV + j0 + j;
#pragma unroll
        for (int m = 0; m < R; ++m) dSg[(size_t)m * DV] = dS[m];
        // rows of Kb dS'; lanes 0-15 keep rows 0-7 of the warp's two row
        // groups, lanes 16-31 rows 8-15
        const bool hi = lane >= 16;
        float pk[C];
#pragma unroll
        for (int r = 0; r < C; ++r) pk[r] = dot_rows<R>(b.kb() + r * DK + i0, dS);
#pragma unroll
        for (int m = 0; m < C / 2; ++m) {
            const float send = hi ? pk[m] : pk[m + 8], keep = hi ? pk[m + 8] : pk[m];
            red[warp][m][lane] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        __syncthreads();
        float du = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) du += red[w][rg & 7][(rg >> 3) * 16 + j];
#pragma unroll
        for (int r2 = 0; r2 < C; ++r2) du = fmaf(b.pm()[r2 * C + rg], xs[it & 1][r2][j], du);  // P^T dO
        us[rg][j] = du;
        p.dUst[idx * C * DV + (size_t)rg * DV + j0 + j] = du;
        if (c > 0) dov = load_do(c - 1);
        __syncthreads();
        // dS <- Diag(gamma_C) dS + Qd^T dO - W^T dU
        const float *gc = b.gc() + i0;
#pragma unroll
        for (int m = 0; m < R; ++m) dS[m] *= gc[m];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            axpy_rows<R>(b.qd() + r * DK + i0, xs[it & 1][r][j], dS);
            axpy_rows<R>(b.w() + r * DK + i0, -us[r][j], dS);
        }
    }
    if (p.ds0) {
#pragma unroll
        for (int m = 0; m < R; ++m) p.ds0[((size_t)nh * DK + i0 + m) * DV + j0 + j] = dS[m];
    }
}

// The two passes are independent (the reverse one needs the prep blocks and
// dO, not the forward states), so one launch runs both: blockIdx.z = 0 the
// forward pass, 1 the reverse pass.
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kChainThreads, 2) chain_kernel(BwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<ChainSm<DK> *>(smem_raw);
    if (blockIdx.z == 0) fwd_chain<DK, DV, T>(p, sm);
    else rev_chain<DK, DV, T>(p, sm);
}

// ---- the per-chunk gradients: one CTA per (chunk, head)
template <int DK, int DV> struct alignas(16) GradSm {
    static constexpr int LK = DK + 4;
    static constexpr int NB = kThreads / DK;   // threads per key channel
    static constexpr int LV = DV + 4;
    PrepSm<DK, DV> pr;                         // its vs holds dV once V is used
    static constexpr int LM = PrepSm<DK, DV>::LM;
    float us[C][LM];                           // U, then dKi
    float dus[C][LV], dos[C][LV];              // dU, dO
    float dqd[C][LK], dw[C][LK], dkb[C][LK];   // dw: dW, then dKd
    float dP[C][C], dT[C][C], M[C][C], dLs[C][C], dA[C][C];
    float dgc[DK];                             // dgamma_C
    float bs[NB][DK], ks[NB][DK];              // per row block: sum of dG, colsum of dKb (.) Kb
};

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kThreads, 2) grad_kernel(BwdParams p) {
    using Sm = GradSm<DK, DV>;
    constexpr int NB = Sm::NB;
    constexpr int RPT = C / NB;  // rows per thread in the row-wise steps
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<Sm *>(smem_raw);
    auto &pr = sm.pr;
    const long slot = blockIdx.x;
    const int h = blockIdx.y, tid = threadIdx.x, H = p.H;
    Seq s;
    int c;
    if (!chunk_of_slot(p, slot, s, c)) return;
    const int t0 = s.bos + c * C, n = min(C, s.len - c * C);
    const size_t idx = (size_t)slot * H + h;
    const T *dy = (const T *)p.dy, *gate = (const T *)p.gate;

    {  // U, dU (workspace) and dO = gate (.) dy; loads first, then the stores
        constexpr int NV = C * DV / kThreads;
        float uv[NV], duv[NV], dov[NV];
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int e = tid + u * kThreads, r = e / DV, jj = e % DV;
            uv[u] = p.Ust[idx * C * DV + e];
            duv[u] = p.dUst[idx * C * DV + e];
            dov[u] = 0.f;
            if (r < n) {
                const size_t o = ((size_t)(t0 + r) * H + h) * DV + jj;
                dov[u] = gate ? ld(dy + o) * ld(gate + o) : ld(dy + o);
            }
        }
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int e = tid + u * kThreads, r = e / DV, jj = e % DV;
            sm.us[r][jj] = uv[u];
            sm.dus[r][jj] = duv[u];
            sm.dos[r][jj] = dov[u];
        }
    }
    // dQd = dO S^T, dW = -dU S^T, dKb = U dS'^T on split-tf32 tensor-core tiles
    // (B[j][i] = S[i][j]); warp w takes key channels 8 w NTG .. 8 (w + 1) NTG - 1;
    // dgamma_C = rowsum(dS' (.) S) from the same operands.  This runs before the
    // chunk's own operands are formed: their shared memory meanwhile stages S
    // and dS' in blocks of 16 columns (cp.async, two blocks in flight).
    {
        constexpr int NTG = DK / 8 / (kThreads / 32);
        constexpr int JB = 16, LS = JB + 4;  // columns per staged block; row stride (floats)
        static_assert(2 * 2 * DK * LS * sizeof(float) <= sizeof(PrepSm<DK, DV>), "staging fits");
        float(*stage)[2][DK][LS] = reinterpret_cast<float(*)[2][DK][LS]>(&pr);  // [buffer][S, dS'][i][j]
        const float *Sb = p.Sst + idx * DK * DV, *Db = p.dSst + idx * DK * DV;
        auto fetch = [&](int blk, int buf) {
            for (int e = tid; e < 2 * DK * JB / 4; e += kThreads) {
                const int m = e / (DK * JB / 4), i = (e / (JB / 4)) % DK, c4 = e % (JB / 4);
                cp_async16(&stage[buf][m][i][4 * c4], (m ? Db : Sb) + (size_t)i * DV + blk * JB + 4 * c4, true);
            }
            cp_async_commit();
        };
        const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
        float aq[NTG][4], aw[NTG][4], ab[NTG][4], ag[NTG];
#pragma unroll
        for (int nt = 0; nt < NTG; ++nt) {
            ag[nt] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) aq[nt][e] = aw[nt][e] = ab[nt][e] = 0.f;
        }
        fetch(0, 0);
        for (int blk = 0; blk < DV / JB; ++blk) {
            cp_async_wait<0>();
            __syncthreads();  // block blk landed; buffer (blk + 1) & 1 is free
            if (blk + 1 < DV / JB) fetch(blk + 1, (blk + 1) & 1);
            const auto &st = stage[blk & 1];
#pragma unroll
            for (int kk = 0; kk < JB / 8; ++kk) {
                const int j = blk * JB + 8 * kk + t, jl = 8 * kk + t;
                uint32_t oh[4], ol[4], dh[4], dl[4], uh[4], ul[4];
                split_tf32(sm.dos[g][j], oh[0], ol[0]);
                split_tf32(sm.dos[g + 8][j], oh[1], ol[1]);
                split_tf32(sm.dos[g][j + 4], oh[2], ol[2]);
                split_tf32(sm.dos[g + 8][j + 4], oh[3], ol[3]);
                split_tf32(sm.dus[g][j], dh[0], dl[0]);
                split_tf32(sm.dus[g + 8][j], dh[1], dl[1]);
                split_tf32(sm.dus[g][j + 4], dh[2], dl[2]);
                split_tf32(sm.dus[g + 8][j + 4], dh[3], dl[3]);
                split_tf32(sm.us[g][j], uh[0], ul[0]);
                split_tf32(sm.us[g + 8][j], uh[1], ul[1]);
                split_tf32(sm.us[g][j + 4], uh[2], ul[2]);
                split_tf32(sm.us[g + 8][j + 4], uh[3], ul[3]);
#pragma unroll
                for (int nt = 0; nt < NTG; ++nt) {
                    const int i = 8 * (warp * NTG + nt) + g;
                    const float s0 = st[0][i][jl], s1 = st[0][i][jl + 4];
                    const float d0 = st[1][i][jl], d1 = st[1][i][jl + 4];
                    ag[nt] = fmaf(s0, d0, fmaf(s1, d1, ag[nt]));
                    mma3(aq[nt], oh, ol, s0, s1);
                    mma3(aw[nt], dh, dl, s0, s1);
                    mma3(ab[nt], uh, ul, d0, d1);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NTG; ++nt) {
            const int ib = 8 * (warp * NTG + nt);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = g + 8 * (e >> 1), i = ib + 2 * t + (e & 1);
                sm.dqd[r][i] = aq[nt][e];
                sm.dw[r][i] = -aw[nt][e];
                sm.dkb[r][i] = ab[nt][e];
            }
            float a = ag[nt];  // row ib + g: the four lanes t hold interleaved columns
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            if (t == 0) sm.dgc[ib + g] = a;  // times gamma_C once the operands are formed
        }
    }
    __syncthreads();  // the staging area becomes the chunk's operands
    prep_chunk<DK, DV, T>(p, pr, h, t0, n);  // ends with a barrier
    __syncthreads();
    {  // dP = tril(dO U^T), dT = dU V^T + dW Kd^T: thread (r, s)
        const int r = tid >> 4, s2 = tid & 15;
        float dp = 0.f, dt = 0.f;
#pragma unroll 8
        for (int c4 = 0; c4 < DV / 4; ++c4) {
            dp = dot4(*reinterpret_cast<const float4 *>(&sm.dos[r][4 * c4]),
                      *reinterpret_cast<const float4 *>(&sm.us[s2][4 * c4]), dp);
            dt = dot4(*reinterpret_cast<const float4 *>(&sm.dus[r][4 * c4]),
                      *reinterpret_cast<const float4 *>(&pr.vs[s2][4 * c4]), dt);
        }
#pragma unroll 8
        for (int c4 = 0; c4 < DK / 4; ++c4)
            dt = dot4(*reinterpret_cast<const float4 *>(&sm.dw[r][4 * c4]),
                      *reinterpret_cast<const float4 *>(&pr.kd[s2][4 * c4]), dt);
        const float dpm = r >= s2 ? dp : 0.f;
        sm.dP[r][s2] = dpm;
        sm.dT[r][s2] = dt;
    }
    __syncthreads();
    {  // M = X^T dT Diag(beta): thread (r, s)
        const int r = tid >> 4, s2 = tid & 15;
        float m = 0.f;
#pragma unroll
        for (int q = 0; q < C; ++q) m = fmaf(pr.X[q][r], sm.dT[q][s2], m);
        sm.M[r][s2] = m * pr.beta[s2];
    }
    for (int e = tid; e < C * DV; e += kThreads) {  // dV = T^T dU into vs (V is used up)
        const int r = e / DV, jj = e % DV;
        float d = 0.f;
#pragma unroll
        for (int q = 0; q < C; ++q) d = fmaf(pr.Tm[q][r], sm.dus[q][jj], d);
        pr.vs[r][jj] = d;
    }
    __syncthreads();
    {  // dL = -M X^T (strictly lower part); dA = Diag(beta) strict(dL): thread (r, s)
        const int r = tid >> 4, s2 = tid & 15;
        float l = 0.f;
#pragma unroll
        for (int q = 0; q < C; ++q) l = fmaf(sm.M[r][q], pr.X[s2][q], l);
        const float ls = r > s2 ? -l : 0.f;
        sm.dLs[r][s2] = ls;
        sm.dA[r][s2] = pr.beta[r] * ls;
    }
    __syncthreads();
    if (tid < n) {  // dbeta = colsum(X (.) dT) + rowsum(strict(dL) (.) A)
        const int r = tid;
        float db = 0.f;
#pragma unroll
        for (int q = 0; q < C; ++q) {
            db = fmaf(pr.X[q][r], sm.dT[q][r], db);
            db = fmaf(sm.dLs[r][q], pr.A[r][q], db);
        }
        p.dbeta[(size_t)(t0 + r) * H + h] = db;
    }
    for (int e = tid; e < C * DV; e += kThreads) {
        const int r = e / DV, jj = e % DV;
        if (r < n) p.dv[((size_t)(t0 + r) * H + h) * DV + jj] = pr.vs[r][jj];
    }
    {  // dKd = T^T dW + dA Ki, dKi = dA^T Kd + dP^T Qd, dQd += dP Ki on split-tf32 tiles
       // (M = the 16 rows, K = 16, N = key channels); warp w takes channels 8 w NTG ..
       // 8 (w + 1) NTG - 1 and writes its results over its own columns: dKd over dW,
       // dKi over U (used up), dQd in place
        constexpr int NTG = DK / 8 / (kThreads / 32);
        const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
        // A fragment of k-tile kt of a 16 x 16 matrix given by an element function:
        // a0 = (g, 8kt + t), a1 = (g + 8, 8kt + t), a2 = (g, 8kt + t + 4), a3 = (g + 8, 8kt + t + 4)
        auto a_frag = [&](auto elem, int kt, uint32_t (&ah)[4], uint32_t (&al)[4]) {
#pragma unroll
            for (int e = 0; e < 4; ++e) split_tf32(elem(g + 8 * (e & 1), 8 * kt + t + 4 * (e >> 1)), ah[e], al[e]);
        };
        auto tT = [&](int r, int q) { return pr.Tm[q][r]; };
        auto dA = [&](int r, int q) { return sm.dA[r][q]; };
        auto dAT = [&](int r, int q) { return sm.dA[q][r]; };
        auto dPT = [&](int r, int q) { return sm.dP[q][r]; };
        auto dPm = [&](int r, int q) { return sm.dP[r][q]; };
        float dkd[NTG][4], dki[NTG][4], dqd[NTG][4];
#pragma unroll
        for (int nt = 0; nt < NTG; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                dkd[nt][e] = dki[nt][e] = 0.f;
                dqd[nt][e] = sm.dqd[g + 8 * (e >> 1)][8 * (warp * NTG + nt) + 2 * t + (e & 1)];
            }
        // B[q][i] = X[q][i]: b0 = X[8kt + t][8nt + g], b1 = X[8kt + t + 4][8nt + g]
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            uint32_t ah[4], al[4];
            const int q0 = 8 * kt + t;
            a_frag(tT, kt, ah, al);
#pragma unroll
            for (int nt = 0; nt < NTG; ++nt) {
                const int i = 8 * (warp * NTG + nt) + g;
                mma3(dkd[nt], ah, al, sm.dw[q0][i], sm.dw[q0 + 4][i]);
            }
            a_frag(dA, kt, ah, al);
#pragma unroll
            for (int nt = 0; nt < NTG; ++nt) {
                const int i = 8 * (warp * NTG + nt) + g;
                mma3(dkd[nt], ah, al, pr.ki[q0][i], pr.ki[q0 + 4][i]);
            }
            a_frag(dAT, kt, ah, al);
#pragma unroll
            for (int nt = 0; nt < NTG; ++nt) {
                const int i = 8 * (warp * NTG + nt) + g;
                mma3(dki[nt], ah, al, pr.kd[q0][i], pr.kd[q0 + 4][i]);
            }
            a_frag(dPT, kt, ah, al);
#pragma unroll
            for (int nt = 0; nt < NTG; ++nt) {
                const int i = 8 * (warp * NTG + nt) + g;
                mma3(dki[nt], ah, al, pr.qd[q0][i], pr.qd[q0 + 4][i]);
            }
            a_frag(dPm, kt, ah, al);
#pragma unroll
            for (int nt = 0; nt < NTG; ++nt) {
                const int i = 8 * (warp * NTG + nt) + g;
                mma3(dqd[nt], ah, al, pr.ki[q0][i], pr.ki[q0 + 4][i]);
            }
        }
        __syncwarp();  // this warp's reads of its dW columns are done
#pragma unroll
        for (int nt = 0; nt < NTG; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = g + 8 * (e >> 1), i = 8 * (warp * NTG + nt) + 2 * t + (e & 1);
                sm.dw[r][i] = dkd[nt][e];
                sm.us[r][i] = dki[nt][e];
                sm.dqd[r][i] = dqd[nt][e];
            }
    }
    __syncthreads();
    {  // dq, dk, dg for rows r0 .. r0 + RPT - 1 of channel i
        const int i = tid % DK, rb = tid / DK, r0 = rb * RPT;
        float dkd[RPT], dki[RPT], dqd[RPT];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            dkd[rr] = sm.dw[r0 + rr][i];
            dki[rr] = sm.us[r0 + rr][i];
            dqd[rr] = sm.dqd[r0 + rr][i];
        }
        float dG[RPT], bsum = 0.f, ksum = 0.f;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int r = r0 + rr;
            const float kb = pr.kb[r][i], dkb = sm.dkb[r][i];
            dG[rr] = dkd[rr] * pr.kd[r][i] - dki[rr] * pr.ki[r][i] + dqd[rr] * pr.qd[r][i] - dkb * kb;
            bsum += dG[rr];
            ksum = fmaf(dkb, kb, ksum);
        }
        sm.bs[rb][i] = bsum;
        sm.ks[rb][i] = ksum;
        __syncthreads();
        // dg_r = dgamma_C gamma_C + colsum(dKb (.) Kb) + sum of dG over rows >= r
        float acc = sm.dgc[i] * pr.gc[i];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            acc += sm.ks[b][i];
            if (b > rb) acc += sm.bs[b][i];
        }
        const float GC = pr.gs[C - 1][i];
#pragma unroll
        for (int rr = RPT - 1; rr >= 0; --rr) {
            const int r = r0 + rr;
            acc += dG[rr];
            if (r < n) {
                const float Gr = pr.gs[r][i], e = expf(Gr);
                const size_t o = ((size_t)(t0 + r) * H + h) * DK + i;
                p.dk[o] = dkd[rr] * e + dki[rr] * expf(-Gr) + sm.dkb[r][i] * expf(GC - Gr);
                p.dq[o] = p.scale * dqd[rr] * e;
                p.dg[o] = acc;
            }
        }
    }
}

// two CTAs of grad_kernel per SM (228 KB of shared memory, 1 KB reserved per CTA)
static_assert(sizeof(GradSm<128, 128>) + 1024 <= 228 * 1024 / 2, "grad_kernel: two CTAs per SM");

template <typename K> cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DK, int DV, typename T>
cudaError_t launch_bwd_t(const BwdParams &p, long slots, cudaStream_t st) {
    static_assert(C * C == kThreads, "prep_kernel writes P with one thread per entry");
    const dim3 per_chunk((unsigned)slots, (unsigned)p.H), per_seq((unsigned)(p.N * p.H), DV / (kHalves * NC), 2);
    cudaError_t e;
    if ((e = set_smem(prep_kernel<DK, DV, T>, sizeof(PrepSm<DK, DV>))) != cudaSuccess) return e;
    if ((e = set_smem(chain_kernel<DK, DV, T>, sizeof(ChainSm<DK>))) != cudaSuccess) return e;
    if ((e = set_smem(grad_kernel<DK, DV, T>, sizeof(GradSm<DK, DV>))) != cudaSuccess) return e;
    if (slots > 0) prep_kernel<DK, DV, T><<<per_chunk, kThreads, sizeof(PrepSm<DK, DV>), st>>>(p);
    chain_kernel<DK, DV, T><<<per_seq, kChainThreads, sizeof(ChainSm<DK>), st>>>(p);
    if (slots > 0) grad_kernel<DK, DV, T><<<per_chunk, kThreads, sizeof(GradSm<DK, DV>), st>>>(p);
    return cudaGetLastError();
}

template <int DK, typename T>
cudaError_t launch_bwd_dk(const BwdParams &p, int dv, long slots, cudaStream_t st) {
    return dv == 128 ? launch_bwd_t<DK, 128, T>(p, slots, st) : launch_bwd_t<DK, 64, T>(p, slots, st);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

long slots_of(long T, long N) { return T / C + N; }

// Workspace regions (bytes, each 256-byte aligned): prep blocks, S, dS', U, dU.
struct WsLayout {
    size_t prep, S, dS, U, dU, total;
};

WsLayout ws_layout(long T, long N, long H, long dk, long dv) {
    const size_t ch = (size_t)slots_of(T, N) * H;
    const size_t blk = 3 * C * dk + C * dv + C * C + dk;
    WsLayout w;
    w.prep = 0;
    w.S = w.prep + align256(ch * blk * sizeof(float));
    w.dS = w.S + align256(ch * dk * dv * sizeof(float));
    w.U = w.dS + align256(ch * dk * dv * sizeof(float));
    w.dU = w.U + align256(ch * C * dv * sizeof(float));
    w.total = w.dU + align256(ch * C * dv * sizeof(float));
    return w;
}

bool ok_dim(int d) { return d == 64 || d == 128; }

}  // namespace
}  // namespace kda

extern "C" {

size_t kda_bwd_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                              int32_t dv) {
    if (total_tokens < 0 || num_seqs < 0 || H < 1 || !kda::ok_dim(dk) || !kda::ok_dim(dv)) return 0;
    return kda::ws_layout(total_tokens, num_seqs, H, dk, dv).total;
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
    if ((long)num_seqs * H > 0x7fffffffL || kda::slots_of(total_tokens, num_seqs) > 0x7fffffffL)
        return KDA_ERR_UNSUPPORTED;
    const size_t need = kda_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if ((uintptr_t)workspace % 256) return KDA_ERR_ALIGNMENT;

    const kda::WsLayout w = kda::ws_layout(total_tokens, num_seqs, H, dk, dv);
    char *ws = (char *)workspace;
    kda::BwdParams p{};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.gate = gate; p.dy = dy;
    p.cu = cu_seqlens;
    p.s0 = initial_state; p.dsT = d_final_state;
    p.dq = dq; p.dk = dk_out; p.dv = dv_out; p.dg = dg; p.dbeta = dbeta; p.dgate = dgate;
    p.ds0 = d_initial_state;
    p.prep = (float *)(ws + w.prep);
    p.Sst = (float *)(ws + w.S);
    p.dSst = (float *)(ws + w.dS);
    p.Ust = (float *)(ws + w.U);
    p.dUst = (float *)(ws + w.dU);
    p.N = num_seqs; p.H = H; p.T = total_tokens;
    p.scale = scale;
    const long slots = total_tokens > 0 ? kda::slots_of(total_tokens, num_seqs) : 0;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    const bool bf = dtype == KDA_DTYPE_BF16;
    if (dk == 128)
        e = bf ? kda::launch_bwd_dk<128, __nv_bfloat16>(p, dv, slots, st)
               : kda::launch_bwd_dk<128, float>(p, dv, slots, st);
    else
        e = bf ? kda::launch_bwd_dk<64, __nv_bfloat16>(p, dv, slots, st)
               : kda::launch_bwd_dk<64, float>(p, dv, slots, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
