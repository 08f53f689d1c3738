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
        header[2] = 0;
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
// 16 state columns:
//   Sin[first]     = initial state (or zeros)
//   Sin[first + 1] = Szero[first]       (piece 0 is summarised from the
//                                         initial state itself, no M needed)
//   Sin[first + j] = M[first + j - 1] Sin[first + j - 1] + Szero[first + j - 1]
// fp32 throughout.  Each M (dk x dk) is staged in shared memory with cp.async,
// the next one loading while the current product runs.  Thread t: column
// t % 16, rows (t / 16) * DK/16 ... + DK/16 - 1.
constexpr int kScanCols = 16;

template <int DK, int DV>
struct ScanSmem {
    float M[2][DK * DK];
    float Sp[DK][kScanCols + 1];
    static constexpr size_t bytes() { return sizeof(float) * (2 * DK * DK + DK * (kScanCols + 1)); }
};

template <int DK, int DV>
__global__ void __launch_bounds__(256) scan_kernel(PrefillParams p) {
    constexpr int RW = DK / 16;  // rows per thread
    extern __shared__ __align__(16) unsigned char scan_smem[];
    ScanSmem<DK, DV> &sm = *reinterpret_cast<ScanSmem<DK, DV> *>(scan_smem);
    const int n = blockIdx.x, h = blockIdx.y;
    const int col = threadIdx.x % kScanCols, rg = threadIdx.x / kScanCols;
    const int c = blockIdx.z * kScanCols + col;
    const int f = p.seq_first[n];
    const int np = p.seq_first[n + 1] - f;
    if (np <= 1 || f + np > p.P_max) return;
    const int H = p.H;
    const size_t SS = (size_t)DK * DV, MS = (size_t)DK * DK;
    const float *init = p.initial_state ? p.initial_state + ((size_t)n * H + h) * SS : nullptr;

    auto load_M = [&](int buf, int piece) {
        const float4 *src = reinterpret_cast<const float4 *>(p.M + ((size_t)piece * H + h) * MS);
        float4 *dst = reinterpret_cast<float4 *>(sm.M[buf]);
        for (int x = threadIdx.x; x < DK * DK / 4; x += 256) {
            const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst + x));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src + x)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    if (np > 2) load_M(0, f + 1);

#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int i = rg * RW + r;
        p.Sin[((size_t)f * H + h) * SS + (size_t)i * DV + c] = init ? init[(size_t)i * DV + c] : 0.f;
        const float z = p.Szero[((size_t)f * H + h) * SS + (size_t)i * DV + c];
        p.Sin[((size_t)(f + 1) * H + h) * SS + (size_t)i * DV + c] = z;
        sm.Sp[i][col] = z;
    }
    // S_zero of the piece the next step adds, loaded one step ahead so that
    // its global-memory latency overlaps the current product
    float zn[RW];
    if (np > 2) {
#pragma unroll
        for (int r = 0; r < RW; ++r) zn[r] = p.Szero[((size_t)(f + 1) * H + h) * SS + (size_t)(rg * RW + r) * DV + c];
    }
    for (int j = 2; j < np; ++j) {
        const int buf = j & 1;
        if (j + 1 < np) {
            load_M(buf ^ 1, f + j);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;\n" ::: "memory");
        }
        __syncthreads();
        const float *Ms = sm.M[buf];
        float acc[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) acc[r] = zn[r];
        if (j + 1 < np) {
#pragma unroll
            for (int r = 0; r < RW; ++r)
                zn[r] = p.Szero[((size_t)(f + j) * H + h) * SS + (size_t)(rg * RW + r) * DV + c];
        }
#pragma unroll 2
        for (int kk = 0; kk < DK; kk += 4) {  // four k at a time: float4 reads of the M rows
            const float s0 = sm.Sp[kk][col], s1 = sm.Sp[kk + 1][col];
            const float s2 = sm.Sp[kk + 2][col], s3 = sm.Sp[kk + 3][col];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const float4 m4 = *reinterpret_cast<const float4 *>(&Ms[(rg * RW + r) * DK + kk]);
                acc[r] = fmaf(m4.x, s0, acc[r]);
                acc[r] = fmaf(m4.y, s1, acc[r]);
                acc[r] = fmaf(m4.z, s2, acc[r]);
                acc[r] = fmaf(m4.w, s3, acc[r]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int i = rg * RW + r;
            sm.Sp[i][col] = acc[r];
            p.Sin[((size_t)(f + j) * H + h) * SS + (size_t)i * DV + c] = acc[r];
        }
    }
}

cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st) {
    plan_kernel<<<1, 1024, 0, st>>>(cu, num_seqs, total_tokens, piece_len, P_max, header,
                                    seq_first, pieces);
    return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t launch_scan_t(const PrefillParams &p, cudaStream_t st) {
    const size_t sm = ScanSmem<DK, DV>::bytes();
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    scan_kernel<DK, DV><<<dim3(p.num_seqs, p.H, DV / kScanCols), 256, sm, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st) {
    if (dk == 128 && dv == 128) return launch_scan_t<128, 128>(p, st);
    if (dk == 128 && dv == 64) return launch_scan_t<128, 64>(p, st);
    if (dk == 64 && dv == 128) return launch_scan_t<64, 128>(p, st);
    return launch_scan_t<64, 64>(p, st);
}

}  // namespace kda
