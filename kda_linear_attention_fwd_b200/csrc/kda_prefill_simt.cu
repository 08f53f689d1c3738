// KDA prefill, fp32 CUDA-core variant of the chunk pass.
//
// Used for fp32 inputs (where bf16 tensor-core operands would not meet fp32
// accuracy) and as the plain, easy-to-read statement of the chunk algebra
// that the tensor-core kernels implement.  One CTA of 256 threads runs one
// piece for one head with the state [DK][NC] resident in shared memory.
//
// For a chunk of C <= 16 tokens with incoming state S (rows = key channels):
//   G    = inclusive cumulative sum of g over the chunk (per channel)
//   Qd   = (scale q) exp(G),  Kd = k exp(G),  Ki = k exp(-G),
//   Kb   = k exp(G_C - G)
//   A    = strictly-lower(Kd Ki^T),  P = lower(Qd Ki^T)
//   Tb   = (I + Diag(beta) A)^-1 Diag(beta)      (unit-lower solve, 16x16)
//   W    = Tb Kd,   U = Tb V - W S
//   O    = Qd S + P U,   y = gate (.) O
//   S   <- Diag(exp(G_C)) S + Kb^T U
// The decay ratios exp(+-G) stay within fp32/bf16 range because a chunk has
// at most 16 tokens and every per-token log-decay is >= ln(0.0067): |G| <= 80
// (prism.simon-ai.net page, section "数值稳定性与 Co-Design：BF16 约束下的衰减控制策略";
// affta.cn page, section "第一关：KDA 解决算得动", on the ~0.67% retention floor).
// Rows past the end of a piece carry k = q = v = beta = g = 0 and therefore
// contribute nothing.
#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {

template <int DK, int NC>
struct SimtSmem {
    static constexpr int LDK = DK + 1;
    static constexpr int L16 = 17;
    static constexpr size_t floats =
        (size_t)DK * NC + 5 * 16 * LDK + 16 * DK + 4 * 16 * NC + 3 * 16 * L16 + 16 + DK + 32;
    static constexpr size_t bytes = floats * sizeof(float);
};

// Runs the chunk recurrence over tokens [t0, t0 + len) of head h.
//   OUT   : produce y (needs q and gate)
//   USE_V : the write uses v (false = the transition part, U0 = 0)
// The state starts as the identity (identity = true), a copy of s_init, or
// zeros, and is written to s_out (if not null) at the end.
template <int DK, int NC, bool OUT, bool USE_V, typename T>
__device__ void simt_piece(const PrefillParams &p, int t0, int len, int h, const float *s_init,
                           bool identity, float *s_out, float *smem, const Snap &snap = Snap()) {
    constexpr int NT = 256;
    using L = SimtSmem<DK, NC>;
    constexpr int LDK = L::LDK, L16 = L::L16;
    const int tid = threadIdx.x;
    const int H = p.H;
    const T *q = (const T *)p.q, *k = (const T *)p.k, *v = (const T *)p.v, *g = (const T *)p.g;
    const T *beta = (const T *)p.beta, *gate = (const T *)p.gate;
    T *out = (T *)p.out;

    float *S = smem;
    float *Qd = S + DK * NC;
    float *Kd = Qd + 16 * LDK;
    float *Ki = Kd + 16 * LDK;
    float *Kb = Ki + 16 * LDK;
    float *W = Kb + 16 * LDK;
    float *Gs = W + 16 * LDK;
    float *V = Gs + 16 * DK;
    float *GT = V + 16 * NC;
    float *U = GT + 16 * NC;
    float *O = U + 16 * NC;
    float *A = O + 16 * NC;
    float *P = A + 16 * L16;
    float *Tb = P + 16 * L16;
    float *bet = Tb + 16 * L16;
    float *gl = bet + 16;
    float *rn = gl + DK;

    for (int idx = tid; idx < DK * NC; idx += NT) {
        const int i = idx / NC, c = idx % NC;
        S[idx] = identity ? (i == c ? 1.f : 0.f) : (s_init ? s_init[idx] : 0.f);
    }

    for (int c0 = 0; c0 < len; c0 += 16) {
        const int rows = min(16, len - c0);
        __syncthreads();
        for (int idx = tid; idx < 16 * DK; idx += NT) {
            const int r = idx / DK, i = idx % DK;
            const bool ok = r < rows;
            const size_t o = ((size_t)(t0 + c0 + r) * H + h) * DK + i;
            Kd[r * LDK + i] = ok ? ld(k + o) : 0.f;
            Gs[r * DK + i] = ok ? g_in(ld(g + o), p.flags) : 0.f;
            if (OUT) Qd[r * LDK + i] = ok ? ld(q + o) : 0.f;
        }
        constexpr int DV = NC;
        for (int idx = tid; idx < 16 * NC; idx += NT) {
            const int r = idx / NC, c = idx % NC;
            const bool ok = r < rows;
            const size_t o = ((size_t)(t0 + c0 + r) * H + h) * DV + c;
            if (USE_V) V[idx] = ok ? ld(v + o) : 0.f;
            if (OUT) GT[idx] = ok ? (gate ? gate_in(ld(gate + o), p.flags) : 1.f) : 0.f;
        }
        if (tid < 16) bet[tid] = tid < rows ? beta_in(ld(beta + (size_t)(t0 + c0 + tid) * H + h), p.flags) : 0.f;
        __syncthreads();
        if (p.flags & FLAG_L2NORM) {
            // warp w: rows 2w and 2w+1 -> rn[r] = 1/|q_r|, rn[16 + r] = 1/|k_r|
            const int lane = tid & 31, w = tid >> 5;
            for (int rr = 0; rr < 2; ++rr) {
                const int r = 2 * w + rr;
                float sq = 0.f, sk = 0.f;
                for (int i = lane; i < DK; i += 32) {
                    const float kv = Kd[r * LDK + i];
                    sk += kv * kv;
                    if (OUT) { const float qv = Qd[r * LDK + i]; sq += qv * qv; }
                }
                sq = warp_sum(sq);
                sk = warp_sum(sk);
                if (lane == 0) {
                    rn[r] = rsqrtf(sq + 1e-6f);
                    rn[16 + r] = rsqrtf(sk + 1e-6f);
                }
            }
            __syncthreads();
        }
        // Per channel: cumulative log-decay and the decayed operands.
        if (tid < DK) {
            const int i = tid;
            float G = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                G += Gs[r * DK + i];
                Gs[r * DK + i] = G;
            }
            const float Gl = G;
            gl[i] = expf(Gl);
#pragma unroll 4
            for (int r = 0; r < 16; ++r) {
                const float Gr = Gs[r * DK + i];
                const float eG = expf(Gr), eN = expf(-Gr), eB = expf(Gl - Gr);
                const float kv = Kd[r * LDK + i] * ((p.flags & FLAG_L2NORM) ? rn[16 + r] : 1.f);
                Kd[r * LDK + i] = kv * eG;
                Ki[r * LDK + i] = kv * eN;
                Kb[r * LDK + i] = kv * eB;
                if (OUT) {
                    const float qv = Qd[r * LDK + i] * ((p.flags & FLAG_L2NORM) ? rn[r] : 1.f) * p.scale;
                    Qd[r * LDK + i] = qv * eG;
                }
            }
        }
        __syncthreads();
        {   // A and P: thread (r, s)
            const int r = tid >> 4, s = tid & 15;
            float a = 0.f, pp = 0.f;
            for (int i = 0; i < DK; ++i) {
                const float kis = Ki[s * LDK + i];
                a += Kd[r * LDK + i] * kis;
                if (OUT) pp += Qd[r * LDK + i] * kis;
            }
            A[r * L16 + s] = s < r ? a : 0.f;
            if (OUT) P[r * L16 + s] = s <= r ? pp : 0.f;
        }
        __syncthreads();
        if (tid < 16) {  // forward substitution, lane j = column j of T
            const int j = tid;
            float col[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc -= bet[r] * A[r * L16 + s] * col[s];
                col[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tb[r * L16 + j] = col[r] * bet[j];
        }
        __syncthreads();
        for (int idx = tid; idx < 16 * DK; idx += NT) {
            const int r = idx / DK, i = idx % DK;
            float w = 0.f;
#pragma unroll
            for (int s = 0; s < 16; ++s) w += Tb[r * L16 + s] * Kd[s * LDK + i];
            W[r * LDK + i] = w;
        }
        __syncthreads();
        for (int idx = tid; idx < 16 * NC; idx += NT) {
            const int r = idx / NC, c = idx % NC;
            float u = 0.f;
            if (USE_V) {
#pragma unroll
                for (int s = 0; s < 16; ++s) u += Tb[r * L16 + s] * V[s * NC + c];
            }
            for (int i = 0; i < DK; ++i) u -= W[r * LDK + i] * S[i * NC + c];
            U[idx] = u;
        }
        __syncthreads();
        if (OUT) {
            for (int idx = tid; idx < 16 * NC; idx += NT) {
                const int r = idx / NC, c = idx % NC;
                float o = 0.f;
                for (int i = 0; i < DK; ++i) o += Qd[r * LDK + i] * S[i * NC + c];
#pragma unroll
                for (int s = 0; s < 16; ++s) o += P[r * L16 + s] * U[s * NC + c];
                O[idx] = o;
            }
            __syncthreads();
        }
        for (int idx = tid; idx < DK * NC; idx += NT) {
            const int i = idx / NC, c = idx % NC;
            float sv = gl[i] * S[idx];
#pragma unroll
            for (int s = 0; s < 16; ++s) sv += Kb[s * LDK + i] * U[s * NC + c];
            S[idx] = sv;
        }
        if (float *sp = snap.at(snap.pos0 + c0 + 16))  // same element mapping as the update
            for (int idx = tid; idx < DK * NC; idx += NT) sp[idx] = S[idx];
        if (OUT) {
            for (int idx = tid; idx < 16 * NC; idx += NT) {
                const int r = idx / NC, c = idx % NC;
                if (r < rows)
                    st(out + ((size_t)(t0 + c0 + r) * H + h) * DV + c, GT[idx] * O[idx]);
            }
        }
    }
    __syncthreads();
    if (s_out)
        for (int idx = tid; idx < DK * NC; idx += NT) s_out[idx] = S[idx];
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) simt_summary_kernel(PrefillParams p) {
    extern __shared__ float smem[];
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
        simt_piece<DK, DV, false, true, T>(p, pc.y, pc.z, h, init, false,
                                           p.Szero + ph * DK * DV, smem);
    } else {
        if (!p.summarize_all && j == 0) return;
        simt_piece<DK, DK, false, false, T>(p, pc.y, pc.z, h, nullptr, true, p.M + ph * DK * DK,
                                            smem);
    }
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) simt_output_kernel(PrefillParams p) {
    extern __shared__ float smem[];
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
    simt_piece<DK, DV, true, true, T>(p, pc.y, pc.z, h, init, false, fin, smem,
                                      make_snap(p, n, h, pc.y, (size_t)DK * DV));
}

template <int DK, int DV, typename T>
static cudaError_t launch_simt_t(const PrefillParams &p, bool summaries, cudaStream_t st) {
    const size_t sm_out = SimtSmem<DK, DV>::bytes;
    const size_t sm_sum = SimtSmem<DK, (DK > DV ? DK : DV)>::bytes;
    cudaError_t e;
    if (summaries) {
        e = cudaFuncSetAttribute(simt_summary_kernel<DK, DV, T>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_sum);
        if (e != cudaSuccess) return e;
        simt_summary_kernel<DK, DV, T><<<dim3((unsigned)(p.P_max * p.H), 2), 256, sm_sum, st>>>(p);
        return cudaGetLastError();
    }
    e = cudaFuncSetAttribute(simt_output_kernel<DK, DV, T>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out);
    if (e != cudaSuccess) return e;
    simt_output_kernel<DK, DV, T><<<dim3((unsigned)(p.P_max * p.H)), 256, sm_out, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_dt(const PrefillParams &p, int dk, int dv, bool summaries,
                                  cudaStream_t st) {
    if (dk == 128 && dv == 128) return launch_simt_t<128, 128, T>(p, summaries, st);
    if (dk == 128 && dv == 64) return launch_simt_t<128, 64, T>(p, summaries, st);
    if (dk == 64 && dv == 128) return launch_simt_t<64, 128, T>(p, summaries, st);
    return launch_simt_t<64, 64, T>(p, summaries, st);
}

cudaError_t launch_prefill_simt(const PrefillParams &p, bool bf16, int dk, int dv, bool summaries,
                                cudaStream_t st) {
    if (bf16) return launch_simt_dt<__nv_bfloat16>(p, dk, dv, summaries, st);
    return launch_simt_dt<float>(p, dk, dv, summaries, st);
}

}  // namespace kda
