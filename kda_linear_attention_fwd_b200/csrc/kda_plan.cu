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
// 32 state columns:
//   Sin[first]     = initial state (or zeros)
//   Sin[first + 1] = Szero[first]       (piece 0 is summarised from the
//                                         initial state itself, no M needed)
//   Sin[first + j] = M[first + j - 1] Sin[first + j - 1] + Szero[first + j - 1]
// fp32 throughout.  Each M (dk x dk) is staged in shared memory in two halves
// of dk/2 key channels by cp.async; while one half is in use the next one is
// in flight, so a step never waits for a whole matrix.  Thread t owns the
// four columns 4 (t % 8) .. + 3 of rows t / 8 + 32 r and updates them with
// packed fp32 pair FMAs.  84 KB of shared memory (dk = 128): two CTAs per SM.
constexpr int kScanCols = 32;
constexpr int kScanThreads = 256;

template <int DK>
struct ScanSmem {
    static constexpr int KH = DK / 2;  // key channels in one half of M
    static constexpr int LD = KH + 4;  // padded row: rows one apart fall in different banks
    float M[2][DK * LD];               // M[:, 0:KH] and M[:, KH:DK]
    float4 Sp[DK][kScanCols / 4];      // the running state, this CTA's columns
    static constexpr size_t bytes() {
        return sizeof(float) * 2 * DK * LD + sizeof(float4) * DK * (kScanCols / 4);
    }
};

KDA_DEVICE float2 fma2(float a, float2 b, float2 c) {
    uint64_t d;
    const float2 aa = make_float2(a, a);
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&aa)), "l"(*reinterpret_cast<const uint64_t *>(&b)),
          "l"(*reinterpret_cast<const uint64_t *>(&c)));
    return *reinterpret_cast<float2 *>(&d);
}

template <int DK, int DV>
__global__ void __launch_bounds__(kScanThreads) scan_kernel(PrefillParams p) {
    constexpr int RW = DK / 32;  // rows per thread
    constexpr int KH = ScanSmem<DK>::KH, LD = ScanSmem<DK>::LD;
    extern __shared__ __align__(16) unsigned char scan_smem[];
    ScanSmem<DK> &sm = *reinterpret_cast<ScanSmem<DK> *>(scan_smem);
    const int n = blockIdx.x, h = blockIdx.y;
    const int cq = threadIdx.x % 8, rg = threadIdx.x / 8;
    const int c = blockIdx.z * kScanCols + 4 * cq;  // first of this thread's four columns
    const int f = p.seq_first[n];
    const int np = p.seq_first[n + 1] - f;
    if (np <= 1 || f + np > p.P_max) return;
    const int H = p.H;
    const size_t SS = (size_t)DK * DV, MS = (size_t)DK * DK;
    const float *init = p.initial_state ? p.initial_state + ((size_t)n * H + h) * SS : nullptr;
    // element (row, c) of the state-sized entry of `piece` in `base`
    auto st_at = [&](size_t piece, int row) { return ((size_t)piece * H + h) * SS + (size_t)row * DV + c; };

    // one half of M of `piece` -> buffer `half` (one cp.async group)
    auto load_half = [&](int piece, int half) {
        const float *src = p.M + ((size_t)piece * H + h) * MS + half * KH;
        float *dst = sm.M[half];
        for (int x = threadIdx.x; x < DK * KH / 4; x += kScanThreads) {
            const int row = x / (KH / 4), c4 = x % (KH / 4);
            const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst + row * LD + 4 * c4));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src + (size_t)row * DK + 4 * c4)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    if (np > 2) {
        load_half(f + 1, 0);
        load_half(f + 1, 1);
    }

#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int row = rg + 32 * r;
        const float4 s0 = init ? *reinterpret_cast<const float4 *>(init + (size_t)row * DV + c)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(p.Sin + st_at(f, row)) = s0;
        const float4 z = *reinterpret_cast<const float4 *>(p.Szero + st_at(f, row));
        *reinterpret_cast<float4 *>(p.Sin + st_at(f + 1, row)) = z;
        sm.Sp[row][cq] = z;
    }
    // S_zero of the piece the next step adds, loaded one step ahead so that
    // its global-memory latency overlaps the current product
    float4 zn[RW];
    if (np > 2) {
#pragma unroll
        for (int r = 0; r < RW; ++r) zn[r] = *reinterpret_cast<const float4 *>(p.Szero + st_at(f + 1, rg + 32 * r));
    }
    for (int j = 2; j < np; ++j) {
        const bool more = j + 1 < np;
        float2 acc[RW][2];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            acc[r][0] = make_float2(zn[r].x, zn[r].y);
            acc[r][1] = make_float2(zn[r].z, zn[r].w);
        }
        if (more) {
#pragma unroll
            for (int r = 0; r < RW; ++r) zn[r] = *reinterpret_cast<const float4 *>(p.Szero + st_at(f + j, rg + 32 * r));
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            // in flight: this half, then the other one or the next step's first
            if (hf == 0 || more) {
                asm volatile("cp.async.wait_group 1;\n" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;\n" ::: "memory");
            }
            __syncthreads();  // the half (and the previous step's state) is visible
            const float *Mh = sm.M[hf];
#pragma unroll 2
            for (int kk = 0; kk < KH; kk += 4) {
                float4 s[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) s[i] = sm.Sp[hf * KH + kk + i][cq];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(Mh + (rg + 32 * r) * LD + kk);
                    const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[r][0] = fma2(mv[i], make_float2(s[i].x, s[i].y), acc[r][0]);
                        acc[r][1] = fma2(mv[i], make_float2(s[i].z, s[i].w), acc[r][1]);
                    }
                }
            }
            __syncthreads();  // every thread is done with this half (and with the state)
            if (more) load_half(f + j, hf);
        }
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int row = rg + 32 * r;
            const float4 v = make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
            sm.Sp[row][cq] = v;
            *reinterpret_cast<float4 *>(p.Sin + st_at(f + j, row)) = v;
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
    const size_t sm = ScanSmem<DK>::bytes();
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    scan_kernel<DK, DV><<<dim3(p.num_seqs, p.H, DV / kScanCols), kScanThreads, sm, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st) {
    if (dk == 128 && dv == 128) return launch_scan_t<128, 128>(p, st);
    if (dk == 128 && dv == 64) return launch_scan_t<128, 64>(p, st);
    if (dk == 64 && dv == 128) return launch_scan_t<64, 128>(p, st);
    return launch_scan_t<64, 64>(p, st);
}

}  // namespace kda
