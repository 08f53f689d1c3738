// KDA prefill: the piece plan and the prefix scan over piece summaries.
#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {

// One CTA of 1024 threads turns cu_seqlens into the piece table.  Each
// sequence of length L gets max(1, ceil(L / piece_len)) pieces, counted from
// its first token; an empty sequence gets one empty piece (it only copies
// the initial state to the final state).  Token ranges are clamped to
// [0, total_tokens] so that malformed offsets can never index out of bounds;
// header[1] is set to 1 when cu_seqlens was found inconsistent.
__global__ void __launch_bounds__(1024)
    plan_kernel(const int32_t *__restrict__ cu, int num_seqs, int total_tokens, int piece_len,
                int P_max, int32_t *header, int32_t *seq_first, int4 *pieces) {
    __shared__ int warp_sums[32];
    __shared__ int carry_s;
    __shared__ int bad_s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) {
        carry_s = 0;
        bad_s = (num_seqs > 0 && (cu[0] != 0 || cu[num_seqs] != total_tokens)) ? 1 : 0;
    }
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + tid;
        int cnt = 0;
        if (n < num_seqs) {
            const int a = cu[n], b = cu[n + 1];
            if (b < a) bad_s = 1;
            const int t0 = min(max(a, 0), total_tokens);
            const int t1 = min(max(b, t0), total_tokens);
            const int len = t1 - t0;
            cnt = len <= 0 ? 1 : (len + piece_len - 1) / piece_len;
        }
        int x = cnt;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int s = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sums[lane] = s;  // inclusive over warps
        }
        __syncthreads();
        const int excl = x - cnt + (wid > 0 ? warp_sums[wid - 1] : 0);
        if (n < num_seqs) seq_first[n] = carry_s + excl;
        __syncthreads();
        if (tid == 0) carry_s += warp_sums[31];
        __syncthreads();
    }
    const int P = carry_s;
    if (tid == 0) {
        seq_first[num_seqs] = P;
        header[0] = min(P, P_max);
        header[1] = bad_s | (P > P_max ? 2 : 0);
    }
    __syncthreads();
    for (int n = tid; n < num_seqs; n += 1024) {
        const int f = seq_first[n], c = seq_first[n + 1] - f;
        const int t0 = min(max(cu[n], 0), total_tokens);
        const int t1 = min(max(cu[n + 1], t0), total_tokens);
        const int len = t1 - t0;
        for (int j = 0; j < c; ++j) {
            if (f + j >= P_max) break;
            const int s = t0 + j * piece_len;
            pieces[f + j] = make_int4(n, s, max(0, min(piece_len, len - j * piece_len)), j);
        }
    }
    for (int p = P + tid; p < P_max; p += 1024) pieces[p] = make_int4(-1, 0, 0, 0);
}

// Prefix scan over the pieces of one sequence, for one head and one block of
// 32 state columns:
//   Sin[first]     = initial state (or zeros)
//   Sin[first + 1] = Szero[first]       (piece 0 is summarised from the
//                                         initial state itself, no M needed)
//   Sin[first + j] = M[first + j - 1] Sin[first + j - 1] + Szero[first + j - 1]
// fp32 throughout.  One warp per DK/8 rows, one lane per column.
template <int DK, int DV>
__global__ void __launch_bounds__(256) scan_kernel(PrefillParams p) {
    constexpr int RW = DK / 8;  // rows per warp
    __shared__ float Sp[DK][33];
    const int n = blockIdx.x, h = blockIdx.y, c = blockIdx.z * 32 + (threadIdx.x & 31);
    const int wid = threadIdx.x >> 5;
    const int f = p.seq_first[n];
    const int np = p.seq_first[n + 1] - f;
    if (np <= 1 || f + np > p.P_max) return;
    const int H = p.H;
    const size_t SS = (size_t)DK * DV, MS = (size_t)DK * DK;
    const float *init = p.initial_state ? p.initial_state + ((size_t)n * H + h) * SS : nullptr;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int i = wid * RW + r;
        p.Sin[((size_t)f * H + h) * SS + (size_t)i * DV + c] = init ? init[(size_t)i * DV + c] : 0.f;
        const float z = p.Szero[((size_t)f * H + h) * SS + (size_t)i * DV + c];
        p.Sin[((size_t)(f + 1) * H + h) * SS + (size_t)i * DV + c] = z;
        Sp[i][threadIdx.x & 31] = z;
    }
    __syncthreads();
    for (int j = 2; j < np; ++j) {
        const size_t pp = (size_t)(f + j - 1) * H + h;
        const float *M = p.M + pp * MS;
        float acc[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            acc[r] = p.Szero[pp * SS + (size_t)(wid * RW + r) * DV + c];
        for (int kk = 0; kk < DK; ++kk) {
            const float s = Sp[kk][threadIdx.x & 31];
#pragma unroll
            for (int r = 0; r < RW; ++r) acc[r] += M[(size_t)(wid * RW + r) * DK + kk] * s;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int i = wid * RW + r;
            Sp[i][threadIdx.x & 31] = acc[r];
            p.Sin[((size_t)(f + j) * H + h) * SS + (size_t)i * DV + c] = acc[r];
        }
        __syncthreads();
    }
}

cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st) {
    plan_kernel<<<1, 1024, 0, st>>>(cu, num_seqs, total_tokens, piece_len, P_max, header,
                                    seq_first, pieces);
    return cudaGetLastError();
}

cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st) {
    const dim3 grid(p.num_seqs, p.H, dv / 32);
    if (dk == 128 && dv == 128) scan_kernel<128, 128><<<grid, 256, 0, st>>>(p);
    else if (dk == 128 && dv == 64) scan_kernel<128, 64><<<grid, 256, 0, st>>>(p);
    else if (dk == 64 && dv == 128) scan_kernel<64, 128><<<grid, 256, 0, st>>>(p);
    else scan_kernel<64, 64><<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
