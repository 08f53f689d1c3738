// KDA decode step: one token per (sequence, head), state updated in place.
//
// Per (n, h), with S the fp32 state [dk][dv] (row i = key channel i):
//   S' = Diag(alpha) S                       (channel-wise forget)
//   a  = S'^T k,  b = S'^T q                 (both in the same pass over S')
//   u  = beta (v - a)                        (delta-rule correction)
//   S  = S' + k u^T                          (corrective write)
//   o  = S^T (scale q) = scale (b + (k.q) u) (read after the write, without
//                                             a second pass over S)
//   y  = gate (.) o                          (full-rank output gate)
// Kimi K3 report explainer (affta.cn), section "第一关：KDA 解决算得动".
//
// The step is a streaming read-modify-write of the state (64 KiB per head at
// dk = dv = 128), so it is bound by HBM bandwidth.  One CTA of 256 threads
// owns one head: a warp covers a row of S with 16-byte vector loads (fully
// coalesced 512-byte rows at dv = 128), each thread holds DK*DV/256 state
// values in registers between the read and the write, so S crosses HBM
// exactly once in each direction.  The reduction over the key channels is
// per-thread partial sums followed by a shared-memory combine across warps.
// EXT compiles in the preprocessing flags other than the q/k norm (beta and
// gate as logits, the decay clamp); the plain call runs without them.
#include "kda_common.cuh"

namespace kda {

template <int DK, int DV, typename T, bool EXT>
__global__ void __launch_bounds__(256, 2)
    decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const T *__restrict__ g, const T *__restrict__ beta,
                       const T *__restrict__ gate, T *__restrict__ out, float *state, float scale,
                       int flags_in) {
    const int flags = EXT ? flags_in : (flags_in & FLAG_L2NORM);
    constexpr int NT = 256;
    constexpr int COLG = DV / 4;       // float4 groups per state row
    constexpr int RPP = NT / COLG;     // rows covered by one pass of the CTA
    constexpr int PASSES = DK / RPP;   // state rows held by each thread
    static_assert(NT % COLG == 0 && DK % RPP == 0, "tile shape");

    __shared__ float sk[DK], sq[DK], salpha[DK];
    __shared__ float sv[DV], sgate[DV], su[DV];
    __shared__ __align__(16) float red_a[RPP][DV];
    __shared__ __align__(16) float red_b[RPP][DV];
    __shared__ float snorm[3];

    const long w = blockIdx.x;  // flattened (n, h)
    const int tid = threadIdx.x;
    const int cg = tid % COLG;
    const int r0 = tid / COLG;
    float4 *S = reinterpret_cast<float4 *>(state + w * (long)(DK * DV));

    // 1. Start streaming the state in before anything else.
    float4 s[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) s[p] = ld_stream(S + (r0 + p * RPP) * COLG + cg);

    // 2. Token vectors.
    for (int i = tid; i < DK; i += NT) {
        sk[i] = ld(k + w * DK + i);
        sq[i] = ld(q + w * DK + i);
        salpha[i] = __expf(g_in(ld(g + w * DK + i), flags));
    }
    for (int j = tid; j < DV; j += NT) {
        sv[j] = ld(v + w * DV + j);
        sgate[j] = gate ? gate_in(ld(gate + w * DV + j), flags) : 1.0f;
    }
    __syncthreads();
    if (tid < 32) {
        // k.q and, when asked, the L2 norms of q and k.
        float kq = 0.f, qq = 0.f, kk = 0.f;
        for (int i = tid; i < DK; i += 32) {
            kq += sk[i] * sq[i];
            qq += sq[i] * sq[i];
            kk += sk[i] * sk[i];
        }
        kq = warp_sum(kq);
        qq = warp_sum(qq);
        kk = warp_sum(kk);
        if (tid == 0) {
            const float rq = (flags & FLAG_L2NORM) ? rsqrtf(qq + 1e-6f) : 1.0f;
            const float rk = (flags & FLAG_L2NORM) ? rsqrtf(kk + 1e-6f) : 1.0f;
            snorm[0] = rq;
            snorm[1] = rk;
            snorm[2] = kq * rq * rk;
        }
    }

    // 3. Forget, then partial S'^T k and S'^T q over this thread's rows.
    float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int i = r0 + p * RPP;
        const float al = salpha[i], ki = sk[i], qi = sq[i];
        s[p].x *= al; s[p].y *= al; s[p].z *= al; s[p].w *= al;
        pa[0] += s[p].x * ki; pa[1] += s[p].y * ki; pa[2] += s[p].z * ki; pa[3] += s[p].w * ki;
        pb[0] += s[p].x * qi; pb[1] += s[p].y * qi; pb[2] += s[p].z * qi; pb[3] += s[p].w * qi;
    }
    *reinterpret_cast<float4 *>(&red_a[r0][cg * 4]) = make_float4(pa[0], pa[1], pa[2], pa[3]);
    *reinterpret_cast<float4 *>(&red_b[r0][cg * 4]) = make_float4(pb[0], pb[1], pb[2], pb[3]);
    __syncthreads();

    // 4. Combine across rows: u and the gated output, one thread per column.
    const float rq = snorm[0], rk = snorm[1], kq = snorm[2];
    for (int j = tid; j < DV; j += NT) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int r = 0; r < RPP; ++r) {
            a += red_a[r][j];
            b += red_b[r][j];
        }
        const float bt = beta_in(ld(beta + w), flags);
        const float u = bt * (sv[j] - a * rk);
        const float o = scale * (b * rq + kq * u);
        st(out + w * DV + j, sgate[j] * o);
        su[j] = u * rk;  // the write uses the normalised key: k_i rk u_j
    }
    __syncthreads();

    // 5. Corrective write and stream the state back out.
    const float4 u4 = *reinterpret_cast<const float4 *>(&su[cg * 4]);
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int i = r0 + p * RPP;
        const float ki = sk[i];
        s[p].x += ki * u4.x; s[p].y += ki * u4.y; s[p].z += ki * u4.z; s[p].w += ki * u4.w;
        st_stream(S + i * COLG + cg, s[p]);
    }
}

template <int DK, int DV, typename T>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const void *gate, void *out, float *state,
                                   long nh, float scale, int flags, cudaStream_t st) {
    if (flags & ~FLAG_L2NORM)
        decode_step_kernel<DK, DV, T, true><<<(unsigned)nh, 256, 0, st>>>(
            (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const T *)beta,
            (const T *)gate, (T *)out, state, scale, flags);
    else
        decode_step_kernel<DK, DV, T, false><<<(unsigned)nh, 256, 0, st>>>(
            (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const T *)beta,
            (const T *)gate, (T *)out, state, scale, flags);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_decode_dt(int dk, int dv, const void *q, const void *k, const void *v,
                                    const void *g, const void *beta, const void *gate, void *out,
                                    float *state, long nh, float scale, int flags, cudaStream_t st) {
    if (dk == 128 && dv == 128)
        return launch_decode_t<128, 128, T>(q, k, v, g, beta, gate, out, state, nh, scale, flags, st);
    if (dk == 128 && dv == 64)
        return launch_decode_t<128, 64, T>(q, k, v, g, beta, gate, out, state, nh, scale, flags, st);
    if (dk == 64 && dv == 128)
        return launch_decode_t<64, 128, T>(q, k, v, g, beta, gate, out, state, nh, scale, flags, st);
    return launch_decode_t<64, 64, T>(q, k, v, g, beta, gate, out, state, nh, scale, flags, st);
}

cudaError_t launch_decode(bool bf16, int dk, int dv, const void *q, const void *k, const void *v,
                          const void *g, const void *beta, const void *gate, void *out,
                          float *state, long nh, float scale, int flags, cudaStream_t st) {
    if (bf16)
        return launch_decode_dt<__nv_bfloat16>(dk, dv, q, k, v, g, beta, gate, out, state, nh,
                                               scale, flags, st);
    return launch_decode_dt<float>(dk, dv, q, k, v, g, beta, gate, out, state, nh, scale, flags, st);
}

}  // namespace kda
