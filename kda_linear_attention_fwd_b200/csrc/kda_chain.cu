// The fold of sub-piece maps into piece maps (the prefill's plans with
// sub-pieces; bf16 inputs, dk = dv = 128) on the tensor cores.  For a piece
// made of sub-pieces s0 .. s0 + m - 1 the map [M | S_zero] is a chain of
// affine steps on the 128 x 256 matrix X = [M | S_zero],
//   X <- M_s X + [0 | S_zero_s],
// the composition of the sub-pieces' maps in token order; the prefix scan then
// runs over whole pieces (the piece states of the prefix scan, Kimi K3 report
// explainer, affta.cn, section "KDA 上下文并行，让上下文的交接变薄", applied
// inside one GPU).  Each product is computed with fp32 accuracy from bf16
// operands by splitting every value into a high and a low bf16 part,
// x = x_hi + x_lo, and forming
//   M X ~ M_hi X_hi + M_hi X_lo + M_lo X_hi
// (the dropped M_lo X_lo is about 2^-16 relative), each product one sequence
// of tcgen05.mma (M = 128, N = 256, K = 16 per instruction) with the fp32 sum
// in tensor memory.
//
// One CTA of 256 threads per (piece, head).  Shared memory: M_hi and M_lo
// K-major (32 KB each), X_hi and X_lo MN-major (64 KB each), in the canonical
// no-swizzle layouts.  Per step: the elected lane of warp 0 issues the 24
// MMAs and commits to an mbarrier; meanwhile every thread loads the next
// step's M into registers; after the (time-bounded) wait, warp w reads rows
// 32 (w % 4) .. + 31 and half w / 4 of the columns of the result from tensor
// memory, adds S_zero_s, and writes the split X back as the next B operand
// (or, after the last step, the fp32 maps to the workspace); then the next M
// is split into shared memory.  A wait that gives up sets bit 1 of the error
// word (the workspace header) and ends the chain.  Each thread owns one row
// (its TMEM lane), so its global accesses are row-strided: the kernel is
// bound by global-load latency (measured: about 14 us per step and wave).
#include "kda_common.cuh"
#include "kda_prefill.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace chain {

using namespace sm100;

constexpr int kD = 128;  // rows of X and both sides of A
constexpr int kThreads = 256;

template <int N>
struct Smem {
    alignas(1024) bf16 a_hi[kD * kD];
    alignas(1024) bf16 a_lo[kD * kD];
    alignas(1024) bf16 x_hi[kD * N];
    alignas(1024) bf16 x_lo[kD * N];
    alignas(8) unsigned long long mbar;
    uint32_t tmem_base;
    int fail;
};
template <int N> constexpr size_t smem_bytes() { return sizeof(Smem<N>) + 1024; }

KDA_DEVICE void split(float x, bf16 &hi, bf16 &lo) {
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// A (row-major fp32 [128][128], global) as 8 float4 pairs per thread:
// unit u = t + 256 i -> row u % 128, columns 8 (u / 128) .. + 7
struct ARegs {
    float4 v[8][2];
};
KDA_DEVICE void load_a(ARegs &r, const float *A) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int u = threadIdx.x + kThreads * i, row = u % kD, c8 = u / kD;
        const float4 *src = reinterpret_cast<const float4 *>(A + (size_t)row * kD + 8 * c8);
        r.v[i][0] = src[0];
        r.v[i][1] = src[1];
    }
}
// -> K-major A_hi / A_lo (rows of one 8-thread phase share a core-matrix group:
// conflict-free 16-byte stores)
template <int N>
KDA_DEVICE void store_a(Smem<N> &sm, const ARegs &r) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int u = threadIdx.x + kThreads * i, row = u % kD, c8 = u / kD;
        const float x[8] = {r.v[i][0].x, r.v[i][0].y, r.v[i][0].z, r.v[i][0].w,
                            r.v[i][1].x, r.v[i][1].y, r.v[i][1].z, r.v[i][1].w};
        alignas(16) bf16 hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) split(x[e], hi[e], lo[e]);
        const uint32_t off = kmaj(row, 8 * c8, kD);
        *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.a_hi) + off) = *reinterpret_cast<uint4 *>(hi);
        *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.a_lo) + off) = *reinterpret_cast<uint4 *>(lo);
    }
}
// 8 consecutive columns n0 .. n0 + 7 of row `row` of X -> MN-major X_hi / X_lo
template <int N>
KDA_DEVICE void store_x8(Smem<N> &sm, int row, int n0, const float (&x)[8]) {
    alignas(16) bf16 hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split(x[e], hi[e], lo[e]);
    const uint32_t off = mnmaj(n0, row, kD);
    *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.x_hi) + off) = *reinterpret_cast<uint4 *>(hi);
    *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.x_lo) + off) = *reinterpret_cast<uint4 *>(lo);
}
// A 128 x 128 block of X0 (row-major fp32 [128][128], or zeros when X is
// null) -> columns n_off .. n_off + 127 of X_hi / X_lo.
template <int N>
KDA_DEVICE void store_x_block(Smem<N> &sm, const float *X, int n_off) {
    for (int u = threadIdx.x; u < kD * (kD / 8); u += kThreads) {
        const int row = u % kD, n0 = 8 * (u / kD);
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (X) {
            const float4 a = *reinterpret_cast<const float4 *>(X + (size_t)row * kD + n0);
            const float4 b = *reinterpret_cast<const float4 *>(X + (size_t)row * kD + n0 + 4);
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
        }
        store_x8(sm, row, n_off + n0, x);
    }
}

// Set-up: TMEM columns for D (N fp32 columns) and the completion barrier.
template <int N>
KDA_DEVICE Smem<N> &setup(unsigned char *raw) {
    Smem<N> &sm = *reinterpret_cast<Smem<N> *>(raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u));
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"((uint32_t)N)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (threadIdx.x == 32) {
        mbar_init(smem_u32(&sm.mbar), 1);
        sm.fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return sm;
}

template <int N>
KDA_DEVICE void teardown(Smem<N> &sm) {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base), "r"((uint32_t)N)
                     : "memory");
}

// Issue D = A X (three split products) and wait for it.  Returns false when
// the bounded wait gave up (then every thread returns false).
template <int N>
KDA_DEVICE bool product(Smem<N> &sm, int step, ARegs *next_a, const float *next_A) {
    fence_async_smem();  // the generic-proxy operand writes become visible to the tensor core
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        if (elect_one_sync()) {
            tc_fence_after();
            constexpr uint32_t ID = idesc_bf16(kD, N, 0, 1);  // A K-major, X MN-major
            const uint64_t ahi = sdesc(smem_u32(sm.a_hi), 128, kD * 16), alo = sdesc(smem_u32(sm.a_lo), 128, kD * 16);
            const uint64_t xhi = sdesc(smem_u32(sm.x_hi), 128, kD * 16), xlo = sdesc(smem_u32(sm.x_lo), 128, kD * 16);
            const uint64_t as[3] = {ahi, ahi, alo}, xs[3] = {xhi, xlo, xhi};
#pragma unroll
            for (int t = 0; t < 3; ++t)
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)  // +256 bytes of K = +16 in the start field
                    tc_mma_ss(sm.tmem_base, as[t] + 16 * kk, xs[t] + 16 * kk, ID, (t > 0 || kk > 0) ? 1u : 0u);
            tc_commit(smem_u32(&sm.mbar));
        }
        __syncwarp();
    }
    if (next_a) load_a(*next_a, next_A);  // the next step's transition, while the MMAs run
    bool ok = mbar_wait(smem_u32(&sm.mbar), step & 1);
    if (!ok) sm.fail = 1;
    tc_fence_after();
    return __syncthreads_or(!ok) == 0;
}

// Read back 32 columns c0 .. c0 + 31 of this thread's row of D.
KDA_DEVICE void read_d32(uint32_t tmem_base, int c0, float (&d)[32]) {
    const int w = threadIdx.x >> 5;
    uint32_t r[32];
    tmem_ld32_wait(tmem_base + ((uint32_t)(32 * (w & 3)) << 16) + (uint32_t)c0, r);
#pragma unroll
    for (int e = 0; e < 32; ++e) d[e] = __uint_as_float(r[e]);
}

// ---------------------------------------------------------------- fold
// One CTA per (piece of the output pass, head); X = [M | S_zero] (N = 256).
__global__ void __launch_bounds__(kThreads, 1) tc_subfold_kernel(SubFoldParams p, int32_t *err) {
    constexpr int N = 2 * kD;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int pi = blockIdx.x, h = blockIdx.y;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    if (j >= np - 1) return;
    const int H = p.H, m = p.sub;
    const int fs = p.seq_first_sub[n], nps = p.seq_first_sub[n + 1] - fs;
    if (fs < 0 || (long)fs + nps > p.P_sub_max || (long)j * m + m > nps) return;  // clamped tables
    const size_t s0 = (size_t)fs + (size_t)j * m;
    const size_t MS = (size_t)kD * kD;
    auto Msub = [&](size_t s) { return p.M_sub + (s * H + h) * MS; };
    auto Zsub = [&](size_t s) { return p.Z_sub + (s * H + h) * MS; };

    Smem<N> &sm = setup<N>(smem_raw);
    // X0 = [M_s0 | Z_s0]; a sequence's first piece has no transition (zeros)
    store_x_block(sm, j > 0 ? Msub(s0) : nullptr, 0);
    store_x_block(sm, Zsub(s0), kD);
    ARegs ar;
    load_a(ar, Msub(s0 + 1));
    store_a(sm, ar);
    const int w = threadIdx.x >> 5, row = 32 * (w & 3) + (threadIdx.x & 31), half = w >> 2;
    for (int t = 1; t < m; ++t) {
        const bool last = t + 1 == m;
        if (!product(sm, t - 1, last ? nullptr : &ar, last ? nullptr : Msub(s0 + t + 1))) break;
        // this thread's row, columns half * 128 .. + 127: + [0 | Z_{s0+t}]
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            const int c0 = half * kD + 32 * cb;
            float d[32];
            read_d32(sm.tmem_base, c0, d);
            if (c0 >= kD) {
                const float4 *z = reinterpret_cast<const float4 *>(Zsub(s0 + t) + (size_t)row * kD + (c0 - kD));
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 zz = z[e4];
                    d[4 * e4] += zz.x; d[4 * e4 + 1] += zz.y; d[4 * e4 + 2] += zz.z; d[4 * e4 + 3] += zz.w;
                }
            }
            if (last) {
                float *dst = c0 < kD ? (j > 0 ? p.M + ((size_t)pi * H + h) * MS + (size_t)row * kD + c0 : nullptr)
                                     : p.Z + ((size_t)pi * H + h) * MS + (size_t)row * kD + (c0 - kD);
                if (dst) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        reinterpret_cast<float4 *>(dst)[e4] = make_float4(d[4 * e4], d[4 * e4 + 1], d[4 * e4 + 2], d[4 * e4 + 3]);
                }
            } else {
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const float x[8] = {d[8 * e8], d[8 * e8 + 1], d[8 * e8 + 2], d[8 * e8 + 3],
                                        d[8 * e8 + 4], d[8 * e8 + 5], d[8 * e8 + 6], d[8 * e8 + 7]};
                    store_x8(sm, row, c0 + 8 * e8, x);
                }
            }
        }
        if (!last) store_a(sm, ar);  // the D reads above are complete (waited loads)
    }
    if (sm.fail && threadIdx.x == 0 && err) atomicOr(err, 1);
    teardown(sm);
}

}  // namespace chain

cudaError_t launch_subfold_tc(const SubFoldParams &p, int32_t *err, cudaStream_t st) {
    if (p.sub < 2) return cudaErrorInvalidValue;
    const size_t sm = chain::smem_bytes<2 * chain::kD>();
    cudaError_t e = cudaFuncSetAttribute(chain::tc_subfold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    chain::tc_subfold_kernel<<<dim3(p.P_max, p.H), chain::kThreads, sm, st>>>(p, err);
    return cudaGetLastError();
}

}  // namespace kda
