// KDA prefill, bf16 tensor-core chunk pass (warp-level MMA, state resident
// in registers).
//
// One CTA runs the 16-token chunk recurrence over one piece of one head.
// The state S (dk x NC, fp32) never leaves the registers of the four state
// warps: warp w holds S^T rows [w*NC/4, (w+1)*NC/4) -- i.e. NC/4 state
// columns -- as m16n8k16 accumulator fragments, and the C-fragment layout of
// those accumulators is exactly the A-fragment layout of the next chunk's
// products, so each chunk only converts them to bf16 in registers.
//
// Per chunk (rows are the chunk's tokens, see kda_prefill_simt.cu for the
// algebra):
//   state warps:  U^T  = V^T Tb^T + S^T (-W)^T        (dv x 16, K = 16 and dk)
//                 O^T  = S^T Qd^T + U^T P^T           (dv x 16)
//                 S^T <- S^T Diag(exp G_C) + U^T Kb    (dv x dk, K = 16)
//                 y    = gate (.) O
//   prep warps:   cumulative decay, Qd / Kd / Ki / Kb (bf16), A = Kd Ki^T and
//                 P = Qd Ki^T (tensor cores), Tb = (I + Diag(beta) A)^-1
//                 Diag(beta) (fp32 forward substitution), W = Tb Kd (tensor
//                 cores); all of it one chunk ahead of the state warps.
// Raw input tiles are prefetched with cp.async one chunk further ahead.
// The prep and state warps hand chunks over through two shared-memory stages
// guarded by named barriers (FULL: prep -> state, EMPTY: state -> prep).
//
// The decay is applied as an absolute-position transform inside the chunk
// (Qd, Kd carry exp(G), Ki carries exp(-G)): prism.simon-ai.net,
// "从架构创新出发：K3的MoE与混合注意力设计", section "数值稳定性与 Co-Design：
// BF16 约束下的衰减控制策略".  With at most 16 tokens and log-decay >= ln 0.0067
// per token (affta.cn K3 explainer, section "第一关：KDA 解决算得动"), |G| <= 80
// and exp(+-G) fit bf16/fp32.  exp(G_r) and exp(G_C - G_r) are built as prefix
// and suffix products of exp(g), one exponential per element.
#include <cstdlib>

#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {
namespace tc {

using bf16 = __nv_bfloat16;

constexpr int kThreads = 256;     // 4 state warps + 4 prep warps
constexpr int kStages = 4;        // one stage per prep warp
constexpr int kPad = 8;           // bf16 row padding: conflict-free ldmatrix
constexpr int kL16 = 16 + kPad;   // row length of the 16 x 16 bf16 tiles

// Named barriers (0 is __syncthreads).  Stage s is filled by prep warp s and
// drained by the four state warps: FULL[s] (prep arrives, state waits) and
// EMPTY[s] (state arrives, prep waits), 32 + 128 threads each.
constexpr int BAR_FULL = 1;       // ids 1..4
constexpr int BAR_EMPTY = 5;      // ids 5..8
constexpr int kBarCount = 160;

KDA_DEVICE uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
KDA_DEVICE void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
KDA_DEVICE void bar_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
KDA_DEVICE uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
KDA_DEVICE float2 unpack_bf16(uint32_t x) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&x);
    return __bfloat1622float2(v);
}
KDA_DEVICE void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
KDA_DEVICE void ldsm4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
KDA_DEVICE void ldsm4t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
KDA_DEVICE void cp_async16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
KDA_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> KDA_DEVICE void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Lane addressing of ldmatrix.x4 for the fragment kinds used here.
//  A operand, row-major [m][k] storage:       row (l&7)+((l>>3)&1)*8, col (l>>4)*8
//  B operand from [n][k] storage (k inner):   n (l&7)+(l>>4)*8,       k ((l>>3)&1)*8
//  B operand from [k][n] storage, .trans:     k (l&7)+((l>>3)&1)*8,   n (l>>4)*8
//  A operand from [k][m] storage, .trans:     k (l&7)+(l>>4)*8,       m ((l>>3)&1)*8
// Results: A -> a0..a3; B -> {r0,r1} = n-tile 0 (k lo, k hi), {r2,r3} = n-tile 1.

template <int DK, int NC>
struct Layout {
    static constexpr int LK = DK + kPad;  // row length of [16][DK] bf16 tiles
    static constexpr int LC = NC + kPad;  // row length of [16][NC] bf16 tiles
    static constexpr int MT = NC / 64;    // m16 tiles per state warp
    static constexpr int CW = NC / 4;     // state columns per state warp
    static constexpr int LY = CW + 4;     // output staging row (fp32)
    struct Raw {                          // cp.async targets of one prep warp
        bf16 q[16 * DK], k[16 * DK], g[16 * DK];
    };
    struct Stage {                        // handed from a prep warp to the state warps
        bf16 qd[16 * LK], kb[16 * LK], wn[16 * LK];
        bf16 v[16 * LC], gate[16 * LC];
        bf16 p[16 * kL16], tb[16 * kL16];
        float gam[DK];
    };
    struct Prep {                         // private to one prep warp
        bf16 kd[16 * LK], ki[16 * LK];
        float A[16 * 17];
        float beta[16];
        float rq[16], rk[16];
    };
    struct All {
        Raw raw[kStages];
        Stage st[kStages];
        Prep pr[kStages];
        float ys[4][16 * LY];
    };
    static constexpr size_t bytes = sizeof(All);
};

// Runs tokens [t0, t0 + len) of head h.  OUT: produce y.  USE_V: the write
// uses v (false: the transition part, U0 = 0).  The state starts as the
// identity, a copy of s_init ([DK][NC] fp32) or zeros and is written to s_out.
template <int DK, int NC, bool OUT, bool USE_V>
__device__ void run_piece(const PrefillParams &p, int t0, int len, int h, const float *s_init,
                          bool identity, float *s_out, unsigned char *smem_raw,
                          const Snap &snap = Snap()) {
    using Lay = Layout<DK, NC>;
    constexpr int LK = Lay::LK, LC = Lay::LC, MT = Lay::MT, CW = Lay::CW, LY = Lay::LY;
    typename Lay::All &sm = *reinterpret_cast<typename Lay::All *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    const int nchunks = (len + 15) / 16;

    if (warp < 4) {
        // ------------------------------------------------------------ state
        const int g8 = lane >> 2, q4 = lane & 3;
        const int jb = warp * CW;  // first state column of this warp
        float s[MT][DK / 8][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int nt = 0; nt < DK / 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = jb + 16 * m + g8 + (e >= 2 ? 8 : 0);
                    const int i = 8 * nt + 2 * q4 + (e & 1);
                    s[m][nt][e] = identity ? (i == j ? 1.f : 0.f)
                                           : (s_init ? s_init[(size_t)i * NC + j] : 0.f);
                }
        bf16 *out = (bf16 *)p.out;
        const bool gate_logits = p.gate && (p.flags & FLAG_GATE_LOGITS);
        for (int c = 0; c < nchunks; ++c) {
            const int stg = c & (kStages - 1);
            bar_sync(BAR_FULL + stg, kBarCount);
            typename Lay::Stage &S = sm.st[stg];
            float u[MT][2][4], o[MT][2][4];
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[m][n][e] = o[m][n][e] = 0.f;
            if (USE_V) {  // U0^T = V^T Tb^T
                uint32_t bt[4];
                ldsm4(bt, &S.tb[((lane & 7) + (lane >> 4) * 8) * kL16 + ((lane >> 3) & 1) * 8]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    uint32_t a[4];
                    ldsm4t(a, &S.v[((lane & 7) + (lane >> 4) * 8) * LC + jb + 16 * m +
                                   ((lane >> 3) & 1) * 8]);
                    mma16816(u[m][0], a, bt[0], bt[1]);
                    mma16816(u[m][1], a, bt[2], bt[3]);
                }
            }
            // U^T += S^T (-W)^T ;  O^T = S^T Qd^T
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t bw[4], bq[4];
                const int n_off = ((lane & 7) + (lane >> 4) * 8) * LK + 16 * kk + ((lane >> 3) & 1) * 8;
                ldsm4(bw, &S.wn[n_off]);
                if (OUT) ldsm4(bq, &S.qd[n_off]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    uint32_t a[4];
                    a[0] = pack_bf16(s[m][2 * kk][0], s[m][2 * kk][1]);
                    a[1] = pack_bf16(s[m][2 * kk][2], s[m][2 * kk][3]);
                    a[2] = pack_bf16(s[m][2 * kk + 1][0], s[m][2 * kk + 1][1]);
                    a[3] = pack_bf16(s[m][2 * kk + 1][2], s[m][2 * kk + 1][3]);
                    mma16816(u[m][0], a, bw[0], bw[1]);
                    mma16816(u[m][1], a, bw[2], bw[3]);
                    if (OUT) {
                        mma16816(o[m][0], a, bq[0], bq[1]);
                        mma16816(o[m][1], a, bq[2], bq[3]);
                    }
                }
            }
            uint32_t ua[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                ua[m][0] = pack_bf16(u[m][0][0], u[m][0][1]);
                ua[m][1] = pack_bf16(u[m][0][2], u[m][0][3]);
                ua[m][2] = pack_bf16(u[m][1][0], u[m][1][1]);
                ua[m][3] = pack_bf16(u[m][1][2], u[m][1][3]);
            }
            if (OUT) {  // O^T += U^T P^T
                uint32_t bp[4];
                ldsm4(bp, &S.p[((lane & 7) + (lane >> 4) * 8) * kL16 + ((lane >> 3) & 1) * 8]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    mma16816(o[m][0], ua[m], bp[0], bp[1]);
                    mma16816(o[m][1], ua[m], bp[2], bp[3]);
                }
            }
            // S^T <- S^T Diag(gamma) + U^T Kb
#pragma unroll
            for (int np = 0; np < DK / 16; ++np) {
                uint32_t bk[4];
                ldsm4t(bk, &S.kb[((lane & 7) + ((lane >> 3) & 1) * 8) * LK + 16 * np +
                                 (lane >> 4) * 8]);
                const float2 ga = *reinterpret_cast<const float2 *>(&S.gam[16 * np + 2 * q4]);
                const float2 gb = *reinterpret_cast<const float2 *>(&S.gam[16 * np + 8 + 2 * q4]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float *x = s[m][2 * np];
                    float *y = s[m][2 * np + 1];
                    x[0] *= ga.x; x[1] *= ga.y; x[2] *= ga.x; x[3] *= ga.y;
                    y[0] *= gb.x; y[1] *= gb.y; y[2] *= gb.x; y[3] *= gb.y;
                    mma16816(s[m][2 * np], ua[m], bk[0], bk[1]);
                    mma16816(s[m][2 * np + 1], ua[m], bk[2], bk[3]);
                }
            }
            if (float *sp = snap.at(snap.pos0 + 16 * (c + 1))) {  // state snapshot after chunk c
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int nt = 0; nt < DK / 8; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = jb + 16 * m + g8 + (e >= 2 ? 8 : 0);
                            const int i = 8 * nt + 2 * q4 + (e & 1);
                            sp[(size_t)i * NC + j] = s[m][nt][e];
                        }
            }
            if (OUT) {
                float *ys = sm.ys[warp];
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int n = 0; n < 2; ++n) {
                        const int t = 8 * n + 2 * q4;
                        const int jl = 16 * m + g8;
                        ys[t * LY + jl] = o[m][n][0];
                        ys[(t + 1) * LY + jl] = o[m][n][1];
                        ys[t * LY + jl + 8] = o[m][n][2];
                        ys[(t + 1) * LY + jl + 8] = o[m][n][3];
                    }
                __syncwarp();
                const int rows = min(16, len - 16 * c);
                // lane -> token row (lane >> 1), half of the warp's columns
                const int r = lane >> 1;
                constexpr int HALF = CW / 2;
                if (r < rows) {
                    const int jl0 = (lane & 1) * HALF;
                    bf16 *dst = out + ((size_t)(t0 + 16 * c + r) * H + h) * NC + jb + jl0;
#pragma unroll
                    for (int v8 = 0; v8 < HALF / 8; ++v8) {
                        const uint4 gv = *reinterpret_cast<const uint4 *>(&S.gate[r * LC + jb + jl0 + 8 * v8]);
                        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jl = jl0 + 8 * v8 + 2 * e;
                            float2 gg = unpack_bf16(gw[e]);
                            if (gate_logits) gg = make_float2(sigmoid_f(gg.x), sigmoid_f(gg.y));
                            pk[e] = pack_bf16(gg.x * ys[r * LY + jl], gg.y * ys[r * LY + jl + 1]);
                        }
                        *reinterpret_cast<uint4 *>(dst + 8 * v8) =
                            make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                __syncwarp();
            }
            bar_arrive(BAR_EMPTY + stg, kBarCount);
        }
        if (s_out) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int nt = 0; nt < DK / 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = jb + 16 * m + g8 + (e >= 2 ? 8 : 0);
                        const int i = 8 * nt + 2 * q4 + (e & 1);
                        s_out[(size_t)i * NC + j] = s[m][nt][e];
                    }
        }
        return;
    }

    // ---------------------------------------------------------------- prep
    // Prep warp pw prepares chunks pw, pw + 4, pw + 8, ... into stage pw.
    const int pw = warp - 4;
    const bf16 *q = (const bf16 *)p.q, *k = (const bf16 *)p.k, *g = (const bf16 *)p.g;
    const bf16 *v = (const bf16 *)p.v, *gate = (const bf16 *)p.gate, *beta = (const bf16 *)p.beta;
    typename Lay::Prep &pr = sm.pr[pw];
    typename Lay::Raw &R = sm.raw[pw];
    typename Lay::Stage &S = sm.st[pw];
    float beta_next = 0.f;

    // q, k, g of chunk c -> this warp's raw buffer (rows past the piece are zero)
    auto issue_raw = [&](int c) {
        const int tc = t0 + 16 * c;
        const int rows = min(16, len - 16 * c);
        constexpr int PK = DK / 8;  // 16-byte pieces per row
#pragma unroll 4
        for (int x = lane; x < 16 * PK; x += 32) {
            const int r = x / PK, cc = x % PK;
            const bool ok = r < rows;
            const size_t off = ((size_t)(ok ? tc + r : t0) * H + h) * DK + cc * 8;
            cp_async16(&R.k[r * DK + cc * 8], k + off, ok);
            cp_async16(&R.g[r * DK + cc * 8], g + off, ok);
            if (OUT) cp_async16(&R.q[r * DK + cc * 8], q + off, ok);
        }
        cp_async_commit();
        beta_next = lane < rows ? beta_in(__bfloat162float(beta[(size_t)(tc + lane) * H + h]), p.flags) : 0.f;
    };
    // v and gate of chunk c -> the stage itself (padded rows)
    auto issue_vg = [&](int c) {
        const int tc = t0 + 16 * c;
        const int rows = min(16, len - 16 * c);
        constexpr int PV = NC / 8;
#pragma unroll 4
        for (int x = lane; x < 16 * PV; x += 32) {
            const int r = x / PV, cc = x % PV;
            const bool ok = r < rows;
            const size_t off = ((size_t)(ok ? tc + r : t0) * H + h) * NC + cc * 8;
            if (USE_V) cp_async16(&S.v[r * LC + cc * 8], v + off, ok);
            if (OUT && gate) cp_async16(&S.gate[r * LC + cc * 8], gate + off, ok);
        }
        cp_async_commit();
    };

    if (pw < nchunks) issue_raw(pw);
    for (int c = pw; c < nchunks; c += kStages) {
        if (c >= kStages) bar_sync(BAR_EMPTY + pw, kBarCount);  // stage free again
        issue_vg(c);
        if (lane < 16) pr.beta[lane] = beta_next;
        cp_async_wait<1>();  // raw q, k, g of chunk c have landed
        __syncwarp();

        if (p.flags & FLAG_L2NORM) {  // 1/|q_r|, 1/|k_r| over the head dimension
            for (int r = 0; r < 16; ++r) {
                float kk = 0.f, qq = 0.f;
                for (int i = lane; i < DK; i += 32) {
                    const float kv = __bfloat162float(R.k[r * DK + i]);
                    kk += kv * kv;
                    if (OUT) {
                        const float qv = __bfloat162float(R.q[r * DK + i]);
                        qq += qv * qv;
                    }
                }
                kk = warp_sum(kk);
                qq = warp_sum(qq);
                if (lane == r) {
                    pr.rk[r] = rsqrtf(kk + 1e-6f);
                    pr.rq[r] = rsqrtf(qq + 1e-6f);
                }
            }
            __syncwarp();
        }

        // 1. decay factors and the decayed bf16 operands; lane owns channel
        //    pairs (2 lane, 2 lane + 1) + 64 x
#pragma unroll
        for (int cp2 = 0; cp2 < DK / 64; ++cp2) {
            const int i = 64 * cp2 + 2 * lane;
            float2 e[16], E[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float2 gg = unpack_bf16(*reinterpret_cast<const uint32_t *>(&R.g[r * DK + i]));
                e[r] = make_float2(__expf(g_in(gg.x, p.flags)), __expf(g_in(gg.y, p.flags)));
            }
            float2 acc = make_float2(1.f, 1.f);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                acc.x *= e[r].x; acc.y *= e[r].y;
                E[r] = acc;
            }
            const float2 El = acc;
            const float2 invEl = make_float2(1.f / El.x, 1.f / El.y);
            *reinterpret_cast<float2 *>(&S.gam[i]) = El;
            float2 F = make_float2(1.f, 1.f);  // exp(G_C - G_r), suffix products
#pragma unroll
            for (int r = 15; r >= 0; --r) {
                float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t *>(&R.k[r * DK + i]));
                if (p.flags & FLAG_L2NORM) { kv.x *= pr.rk[r]; kv.y *= pr.rk[r]; }
                *reinterpret_cast<uint32_t *>(&pr.kd[r * LK + i]) = pack_bf16(kv.x * E[r].x, kv.y * E[r].y);
                *reinterpret_cast<uint32_t *>(&pr.ki[r * LK + i]) =
                    pack_bf16(kv.x * (F.x * invEl.x), kv.y * (F.y * invEl.y));
                *reinterpret_cast<uint32_t *>(&S.kb[r * LK + i]) = pack_bf16(kv.x * F.x, kv.y * F.y);
                if (OUT) {
                    float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t *>(&R.q[r * DK + i]));
                    float sc = p.scale;
                    if (p.flags & FLAG_L2NORM) sc *= pr.rq[r];
                    *reinterpret_cast<uint32_t *>(&S.qd[r * LK + i]) =
                        pack_bf16(qv.x * sc * E[r].x, qv.y * sc * E[r].y);
                }
                F.x *= e[r].x; F.y *= e[r].y;
            }
        }
        if (OUT && !gate) {
            const uint32_t one = pack_bf16(1.f, 1.f);
            for (int x = lane; x < 16 * NC / 8; x += 32) {
                const int r = x / (NC / 8), cc = x % (NC / 8);
                *reinterpret_cast<uint4 *>(&S.gate[r * LC + cc * 8]) = make_uint4(one, one, one, one);
            }
        }
        __syncwarp();
        // the raw buffer is free: prefetch this warp's next chunk
        if (c + kStages < nchunks) issue_raw(c + kStages);

        // 2. A = Kd Ki^T (strictly lower, fp32) and P = Qd Ki^T (lower, bf16)
#pragma unroll
        for (int which = 0; which < (OUT ? 2 : 1); ++which) {
            const bf16 *Aop = which == 0 ? pr.kd : S.qd;
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t a[4], b[4];
                ldsm4(a, &Aop[((lane & 7) + ((lane >> 3) & 1) * 8) * LK + 16 * kk + (lane >> 4) * 8]);
                ldsm4(b, &pr.ki[((lane & 7) + (lane >> 4) * 8) * LK + 16 * kk + ((lane >> 3) & 1) * 8]);
                mma16816(acc0, a, b[0], b[1]);
                mma16816(acc1, a, b[2], b[3]);
            }
            const int r0 = lane >> 2, c0 = 2 * (lane & 3);
            const float vals[8] = {acc0[0], acc0[1], acc0[2], acc0[3],
                                   acc1[0], acc1[1], acc1[2], acc1[3]};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int r = r0 + ((e & 2) ? 8 : 0);
                const int sc = c0 + (e & 1) + ((e & 4) ? 8 : 0);
                if (which == 0) {
                    pr.A[r * 17 + sc] = sc < r ? vals[e] : 0.f;
                } else {
                    S.p[r * kL16 + sc] = __float2bfloat16_rn(sc <= r ? vals[e] : 0.f);
                }
            }
        }
        __syncwarp();

        // 3. Tb = (I + Diag(beta) A)^-1 Diag(beta): forward substitution.
        //    Lane j < 16 owns column j; after row r is final it is pushed into
        //    the partial sums of every later row (independent updates).
        if (lane < 16) {
            const int j = lane;
            float col[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) col[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                // col[r] is final here: delta_rj - beta_r sum_{s<r} A[r][s] col[s]
#pragma unroll
                for (int r2 = r + 1; r2 < 16; ++r2)
                    col[r2] -= pr.beta[r2] * pr.A[r2 * 17 + r] * col[r];
            }
            const float bj = pr.beta[j];
#pragma unroll
            for (int r = 0; r < 16; ++r) S.tb[r * kL16 + j] = __float2bfloat16_rn(col[r] * bj);
        }
        __syncwarp();

        // 4. W = Tb Kd -> the stage holds -W (bf16)
        {
            uint32_t a[4];
            ldsm4(a, &S.tb[((lane & 7) + ((lane >> 3) & 1) * 8) * kL16 + (lane >> 4) * 8]);
#pragma unroll
            for (int np = 0; np < DK / 16; ++np) {
                const int n0 = 16 * np;
                uint32_t b[4];
                ldsm4t(b, &pr.kd[((lane & 7) + ((lane >> 3) & 1) * 8) * LK + n0 + (lane >> 4) * 8]);
                float w0[4] = {0.f, 0.f, 0.f, 0.f}, w1[4] = {0.f, 0.f, 0.f, 0.f};
                mma16816(w0, a, b[0], b[1]);
                mma16816(w1, a, b[2], b[3]);
                const int r = lane >> 2, cc = n0 + 2 * (lane & 3);
                *reinterpret_cast<uint32_t *>(&S.wn[r * LK + cc]) = pack_bf16(-w0[0], -w0[1]);
                *reinterpret_cast<uint32_t *>(&S.wn[(r + 8) * LK + cc]) = pack_bf16(-w0[2], -w0[3]);
                *reinterpret_cast<uint32_t *>(&S.wn[r * LK + cc + 8]) = pack_bf16(-w1[0], -w1[1]);
                *reinterpret_cast<uint32_t *>(&S.wn[(r + 8) * LK + cc + 8]) = pack_bf16(-w1[2], -w1[3]);
            }
        }
        // v and gate of chunk c have landed (the raw prefetch may still run)
        if (c + kStages < nchunks) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncwarp();
        bar_arrive(BAR_FULL + pw, kBarCount);
    }
    // consume the state warps' EMPTY arrival for this warp's last chunk
    if (pw < nchunks) bar_sync(BAR_EMPTY + pw, kBarCount);
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) summary_kernel(PrefillParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    // (piece, head) pairs with the head fastest: co-resident CTAs cover all
    // heads of a few pieces, spreading their rows over every memory channel
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    if (!p.summarize_all && j >= np - 1) return;
    const size_t ph = (size_t)pi * p.H + h;
    if (blockIdx.y == 0) {
        const float *init = (j == 0 && p.initial_state)
                                ? p.initial_state + ((size_t)n * p.H + h) * DK * DV
                                : nullptr;
        run_piece<DK, DV, false, true>(p, pc.y, pc.z, h, init, false, p.Szero + ph * DK * DV, smem);
    } else {
        if (!p.summarize_all && j == 0) return;
        run_piece<DK, DK, false, false>(p, pc.y, pc.z, h, nullptr, true, p.M + ph * DK * DK, smem);
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) output_kernel(PrefillParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    // (piece, head) pairs with the head fastest: co-resident CTAs cover all
    // heads of a few pieces, spreading their rows over every memory channel
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    const size_t nh = (size_t)n * p.H + h;
    const float *init = (np == 1) ? (p.initial_state ? p.initial_state + nh * DK * DV : nullptr)
                                  : p.Sin + ((size_t)pi * p.H + h) * DK * DV;
    float *fin = (j == np - 1 && p.final_state) ? p.final_state + nh * DK * DV : nullptr;
    run_piece<DK, DV, true, true>(p, pc.y, pc.z, h, init, false, fin, smem,
                                  make_snap(p, n, h, pc.y, (size_t)DK * DV));
}

template <int DK, int DV>
static cudaError_t launch_t(const PrefillParams &p, bool summaries, cudaStream_t st) {
    cudaError_t e;
    if (summaries) {
        const size_t sm = Layout<DK, DV>::bytes > Layout<DK, DK>::bytes ? Layout<DK, DV>::bytes
                                                                        : Layout<DK, DK>::bytes;
        e = cudaFuncSetAttribute(summary_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sm);
        if (e != cudaSuccess) return e;
        summary_kernel<DK, DV><<<dim3((unsigned)(p.P_max * p.H), 2), kThreads, sm, st>>>(p);
        return cudaGetLastError();
    }
    const size_t sm = Layout<DK, DV>::bytes;
    e = cudaFuncSetAttribute(output_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm);
    if (e != cudaSuccess) return e;
    output_kernel<DK, DV><<<dim3((unsigned)(p.P_max * p.H)), kThreads, sm, st>>>(p);
    return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_prefill_simt(const PrefillParams &p, bool bf16, int dk, int dv, bool summaries,
                                cudaStream_t st);

cudaError_t launch_prefill_tc(const PrefillParams &p, int dk, int dv, bool summaries,
                              cudaStream_t st) {
    if (dk == 128 && dv == 128) return tc::launch_t<128, 128>(p, summaries, st);
    if (dk == 128 && dv == 64) return tc::launch_t<128, 64>(p, summaries, st);
    if (dk == 64 && dv == 128) return tc::launch_t<64, 128>(p, summaries, st);
    return tc::launch_t<64, 64>(p, summaries, st);
}

cudaError_t launch_prefill_tc5(const PrefillParams &p, bool summaries, cudaStream_t st);
cudaError_t launch_prefill_c32(const PrefillParams &p, bool summaries, cudaStream_t st);

// The chunk pass for one call.  bf16 inputs run on the tensor cores: for
// dk = dv = 128 the 32-token tcgen05 kernels (plain calls) or the 16-token
// tcgen05 kernels (extended features), the warp-level MMA kernel for the other
// head sizes.  fp32 inputs run the fp32 CUDA-core kernel (bf16 operands would
// not reach fp32 accuracy).  KDA_PREFILL_IMPL=c32|tc5|mma|simt forces a kernel
// where it applies.
cudaError_t launch_prefill_chunks(const PrefillParams &p, bool bf16, int dk, int dv,
                                  bool summaries, cudaStream_t st) {
    const int forced = prefill_impl_forced();
    if (!bf16 || forced == 4) return launch_prefill_simt(p, bf16, dk, dv, summaries, st);
    if (chunk32_eligible(bf16, dk, dv, p.flags, p.snap_tokens) && p.piece_len % 32 == 0)
        return launch_prefill_c32(p, summaries, st);
    if (forced != 3 && dk == 128 && dv == 128) return launch_prefill_tc5(p, summaries, st);
    return launch_prefill_tc(p, dk, dv, summaries, st);
}

}  // namespace kda
