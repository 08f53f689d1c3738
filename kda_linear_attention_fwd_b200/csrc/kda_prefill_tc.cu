// KDA prefill, 16-token chunk pass with the state contractions on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// One CTA runs one piece of one head (dk = dv = 128).  Warps 0-3 form the
// state warpgroup: thread j owns state column j -- row j of S^T -- which
// lives in TMEM lane j (fp32, plus a bf16 copy as an MMA operand).  Per chunk
// (see kda_prefill_simt.cu for the algebra), with everything the chunk needs
// prepared ahead by the prep team:
//
//   MMA 1  D1      = V^T [Tb^T | 0]             (M=128, N=32, K=16; A MN-major smem)
//   MMA 2  D1     += S^T [-W^T | Qd^T]          (K=128; A = bf16 S^T in TMEM)
//          -> D1[:, 0:16] = U^T, D1[:, 16:32] = (Qd S)^T
//   WG     (while MMA 1/2 run) S^T scaled in place by the chunk's exp(G_C)
//          (the plain kernels; the others scale it at the end of the previous chunk);
//          y = gate (.) O of the previous chunk
//   WG     U^T (bf16) -> shared memory (A operand of the next two)
//   MMA 3  S^T    += U^T Kb                     (M=128, N=128, K=16)
//   MMA 4  D1[16:] += U^T P^T                   (M=128, N=16, K=16) -> O^T
//   WG     the bf16 copy of S^T for the next chunk's MMA 2
//
// One elected lane issues the MMAs; tcgen05.commit arrives on an mbarrier that
// the warpgroup waits on with a time bound (2 s): a wait that gives up records
// an error in the workspace header and the kernel drains without further
// tensor work, keeping every named-barrier hand-off so that no warp is left
// waiting.
//
// The prep team (the four warps after the state warps: a decay pair and a
// matrix pair, interleaved over the SM sub-partitions in the plain kernels)
// prepares one chunk at a time into one of three stages: TMA loads of q, k, g
// up to three chunks ahead into a ring of raw tiles (128-byte swizzle) and
// cp.async of v into the stage; exp(G) as prefix and suffix products of
// exp(g), one decay thread per key-channel pair over the 16 rows, rewriting
// the raw tiles in place into Qd, Kd and Ki and writing Kb^T; the Gram
// matrices A = Kd Ki^T and
// P = Qd Ki^T on the two matrix warps in parallel (16x16 tiles are far below
// the smallest tcgen05 tile, so these use warp-level MMA); the 16x16
// unit-lower solve in fp32 on one warp; W = Tb Kd split over the two matrix
// warps by key channel.  Every MMA operand the prep writes is in the
// canonical no-swizzle K-major / MN-major layout.  A stage goes back to the
// team as soon as the update MMAs that read it have completed.
//
// Sources: the token pipeline and the decay floor -- affta.cn K3 explainer,
// section "第一关：KDA 解决算得动"; decay as an absolute-position transform over a
// 16-token tile -- prism.simon-ai.net, "从架构创新出发：K3的MoE与混合注意力设计",
// section "数值稳定性与 Co-Design：BF16 约束下的衰减控制策略"; the split into
// parallel per-chunk preparation and a sequential state pass -- affta.cn page,
// section "FlashKDA ，让线性计算也能沾上并行的光".
#include "kda_common.cuh"
#include "kda_prefill.cuh"
#include "kda_sm100.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <type_traits>

namespace kda {
namespace tc5 {

using namespace sm100;

constexpr int kStages = 3;     // prepared chunks in flight: chunk c -> stage c % 3
constexpr int kRaw = 3;        // q, k, g tiles in flight: chunk c -> raw[c % 3]
// A CTA has NWG state warpgroups (1, or 2 in the paired summary kernel: the
// zero-start state and the transition of one piece, sharing one preparation),
// then the decay pair and the matrix pair.
constexpr int kPair = 64;      // threads of the decay pair and of the matrix pair
template <int NWG> constexpr int kThreadsOf = 128 * NWG + 2 * kPair;
constexpr int kThreads = kThreadsOf<1>;
constexpr int kBlocksPerSM = 2;
constexpr int BAR_FULL = 1;    // ids 1..3: the matrix pair arrives, the state warpgroups wait
constexpr int BAR_EMPTY = 4;   // ids 4..6: the state warpgroups arrive, the decay pair waits
constexpr int BAR_WG = 7;      // state warpgroup 0 only
constexpr int BAR_DEC = 8;     // ids 8..10: the decay pair arrives, the matrix pair waits
constexpr int BAR_DPAIR = 11;  // decay pair only
constexpr int BAR_MPAIR = 12;  // matrix pair only
constexpr int BAR_WG2 = 13;    // state warpgroup 1 only
template <int NWG> constexpr int kBarCountOf = 128 * NWG + kPair;  // FULL and EMPTY
constexpr int kDecCount = 2 * kPair;
constexpr int NC = 128;        // state columns = TMEM lanes = MMA M
constexpr uint32_t kTmemColsPerWG = 256;
constexpr int kAT = 20;        // row stride of the solve's AT matrix: the Gram epilogue's
                               // scattered stores fall in distinct banks

// TMA descriptors of q, k and g as [T][H][128] bf16 (3-D: channel, head,
// token); one box = 64 channels x 1 head x 16 tokens, 128-byte swizzle.
struct TmaMaps {
    CUtensorMap q, k, g;
};

// Byte offset of element (r, ch) of a 16 x 128 bf16 tile that TMA wrote as two
// 64-channel boxes with the 128-byte swizzle: 16-byte chunk j of row r lands
// in chunk j ^ (r & 7) of that row (each box 1024-byte aligned).
KDA_DEVICE uint32_t sw128(int r, int ch) {
    return (uint32_t)((ch >> 6) * 2048 + r * 128 + ((((ch & 63) >> 3) ^ (r & 7)) << 4) + ((ch & 7) << 1));
}

template <int DK, int NWG = 1>
struct Layout {
    // TMEM columns of one state warpgroup (256 of the SM's 512; warpgroup i
    // adds 256 i)
    static constexpr uint32_t COL_S = 0;          // S^T, fp32: DK columns (MMA 3 accumulator)
    static constexpr uint32_t COL_D1 = DK;        // 2 x [U^T | O^T]: 2 x 32 fp32 columns
    static constexpr uint32_t COL_AS = DK + 64;   // bf16 S^T (MMA A operand): DK/2 columns
    static_assert(COL_AS + DK / 2 <= kTmemColsPerWG, "TMEM budget");
    static_assert(DK == 128, "one tile row = two 64-channel TMA boxes");
    struct Raw {                                  // TMA targets (swizzled), overwritten in place:
        alignas(1024) unsigned char q[16 * DK * 2];  //   q -> Qd
        alignas(1024) unsigned char k[16 * DK * 2];  //   k -> Kd
        alignas(1024) unsigned char g[16 * DK * 2];  //   g -> Ki
    };
    struct Stage {
        alignas(16) bf16 b1[32 * DK];   // K-major [32][DK]: rows 0-15 = -W, 16-31 = Qd
        alignas(16) bf16 b0[32 * 16];   // K-major [32][16]: rows 0-15 = Tb, 16-31 = 0
        alignas(16) bf16 b2[DK * 16];   // K-major [DK][16]: Kb^T
        alignas(16) bf16 b3[16 * 16];   // K-major [16][16]: P
        alignas(16) bf16 v[NC * 16];    // MN-major [NC][16]: V^T as the A operand
        alignas(16) float gam[DK];      // exp(G_C) per key channel
    };
    struct Prep {
        alignas(16) float AT[16 * kAT];  // AT[s][r] = beta_r A[r][s], r > s (matrix pair)
        float beta[kStages][16];        // beta of the chunk in each stage
        float nk[2][16], nq[2][16];     // per decay warp and row: partial sums of k^2, q^2
        float rk[16], rq[16];           // 1/|k_r| and scale/|q_r| of the chunk being decayed
    };
    struct All {
        Raw raw[kRaw];
        Stage st[kStages];
        Prep pr;
        alignas(16) bf16 au[NWG][NC * 16];  // K-major [NC][16]: U^T as the A operand
        alignas(16) bf16 io[2][16 * NC];  // gate tile in, y tile out (row-major [16][NC])
        alignas(8) unsigned long long mbar[2 * NWG];
        alignas(8) unsigned long long mbar_raw[kRaw];  // TMA completion of raw[i]
        uint32_t tmem_base;
    };
    // plus slack to align the start to 1024 bytes (the swizzle's period)
    static constexpr size_t bytes = sizeof(All) + 1024;
};

template <typename T>
KDA_DEVICE T *at_bytes(T *base, uint32_t off) {
    return reinterpret_cast<T *>(reinterpret_cast<unsigned char *>(base) + off);
}

// Runs tokens [t0, t0 + len) of head h (see the file comment).  OUT: produce
// y.  USE_V: the write uses v (false: the transition part, U0 = 0).  The
// state starts as the identity, a copy of s_init ([DK][NC] fp32) or zeros and
// is written to s_out.  The fp32 state lives in tensor memory.
// NWG = 2 (summary only): warpgroup 0 runs the zero-start state (from s_init)
// into s_out, warpgroup 1 the transition (identity start) into s_out2; a
// warpgroup with active[i] false takes part in every hand-off but computes
// nothing.
// EXT: the extended entry points' features (beta / gate logits, the decay
// clamp, state snapshots) are compiled in; the plain calls run without them.
template <int DK, bool OUT, bool USE_V, bool L2N, bool EXT, int NWG = 1>
__device__ void run_piece(const PrefillParams &p, const TmaMaps &maps, int t0, int len, int h,
                          const float *s_init, bool identity, float *s_out, unsigned char *smem_raw,
                          const Snap &snap = Snap(), float *s_out2 = nullptr, bool active0 = true,
                          bool active1 = true) {
    static_assert(NWG == 1 || (NWG == 2 && !OUT && USE_V), "paired warpgroups: summaries only");
    using Lay = Layout<DK, NWG>;
    constexpr int kBarCount = kBarCountOf<NWG>;
    const int flags = EXT ? p.flags : 0;  // bits other than the norm switch
    constexpr uint32_t kTmemCols = kTmemColsPerWG * NWG;
    typename Lay::All &sm = *reinterpret_cast<typename Lay::All *>(
        smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    const int nchunks = (len + 15) / 16;
    // decay and matrix warps alternate over the warp slots (plain kernels)
    constexpr bool kInterleave = !L2N && !EXT;

    // ---- set-up: TMEM columns and the two MMA-completion barriers
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 32) {
        for (int i = 0; i < 2 * NWG; ++i) mbar_init(smem_u32(&sm.mbar[i]), 1);
        for (int i = 0; i < kRaw; ++i) mbar_init(smem_u32(&sm.mbar_raw[i]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp < 4 * NWG) {
        // ------------------------------------------------------ state warpgroup
        const int wgi = warp >> 2;                // which state warpgroup
        const int j = tid - 128 * wgi;            // state column = TMEM lane
        const int wwarp = warp & 3;               // warp within the group = TMEM lane quarter
        const bool use_v = USE_V && wgi == 0;     // the transition part has no v
        if (NWG == 2 && wgi == 1) {               // the transition: identity start
            identity = true;
            s_init = nullptr;
            s_out = s_out2;
        }
        const bool active = wgi == 0 ? active0 : active1;
        const int bar_wg = wgi == 0 ? BAR_WG : BAR_WG2;
        const uint32_t colb = kTmemColsPerWG * wgi;
        const uint32_t lane_off = (uint32_t)(wwarp * 32) << 16;
        const uint32_t t_s = tbase + colb + lane_off + Lay::COL_S;
        const uint32_t t_d1 = tbase + colb + lane_off + Lay::COL_D1;
        const uint32_t t_as = tbase + colb + lane_off + Lay::COL_AS;
        const uint32_t mb1 = smem_u32(&sm.mbar[2 * wgi]), mb2 = smem_u32(&sm.mbar[2 * wgi + 1]);
        bf16 *au = sm.au[wgi];
        constexpr int N1 = OUT ? 32 : 16;
        constexpr uint32_t ID_U0 = idesc_bf16(128, N1, 1, 0);
        constexpr uint32_t ID_WS = idesc_bf16(128, N1, 0, 0);
        constexpr uint32_t ID_UK = idesc_bf16(128, DK, 0, 0);
        constexpr uint32_t ID_UP = idesc_bf16(128, 16, 0, 0);
        const bf16 *gate = (const bf16 *)p.gate;
        bf16 *out = (bf16 *)p.out;
        const bool gate_logits = gate && (flags & FLAG_GATE_LOGITS);

        bool ok = active;
        // gate of this thread's column for the chunk whose output is pending;
        // loaded one chunk ahead so the loads are off the critical path
        // gate tile of chunk c -> io[c & 1] (two 16-byte pieces per thread)
        auto load_gate = [&](int c) {
            const int rows = min(16, len - 16 * c);
            bf16 *tile = sm.io[c & 1];
#pragma unroll
            for (int x2 = 0; x2 < 2; ++x2) {
                const int x = j + 128 * x2;
                const int r = x >> 4, cc = x & 15;
                const bool okr = gate && r < rows;
                const size_t off = ((size_t)(okr ? t0 + 16 * c + r : t0) * H + h) * NC + cc * 8;
                if (gate) {
                    cp_async16(&tile[r * NC + cc * 8], gate + off, okr);
                } else {
                    const uint32_t one = pack_bf16(1.f, 1.f);
                    *reinterpret_cast<uint4 *>(&tile[r * NC + cc * 8]) = make_uint4(one, one, one, one);
                }
            }
            cp_async_commit();
        };
        // y = gate (.) O of chunk c: column j of the tile, in place
        auto finish_chunk = [&](int c) {
            if (OUT && ok) {
                uint32_t o[16];
                tmem_ld16_wait(t_d1 + 32 * (c & 1) + 16, o);
                bf16 *tile = sm.io[c & 1];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    float gv = __bfloat162float(tile[t * NC + j]);
                    if (gate_logits) gv = sigmoid_fast(gv);
                    tile[t * NC + j] = __float2bfloat16_rn(gv * __uint_as_float(o[t]));
                }
            }
        };
        // the y tile of chunk c -> global (after a warpgroup barrier)
        auto store_y = [&](int c) {
            const int rows = min(16, len - 16 * c);
            const bf16 *tile = sm.io[c & 1];
#pragma unroll
            for (int x2 = 0; x2 < 2; ++x2) {
                const int x = j + 128 * x2;
                const int r = x >> 4, cc = x & 15;
                if (r < rows)
                    *reinterpret_cast<uint4 *>(out + ((size_t)(t0 + 16 * c + r) * H + h) * NC + cc * 8) =
                        *reinterpret_cast<const uint4 *>(&tile[r * NC + cc * 8]);
            }
        };
        // One pass over the fp32 state (from TMEM, or the initial state when
        // from_init): its bf16 copy becomes the A operand of the next chunk's
        // MMA 2 (not needed after the last chunk, which writes the final state
        // instead), and with gam_next the fp32 state is stored back scaled by
        // that chunk's exp(G_C), so that its MMA 3 accumulates U^T Kb straight
        // into it.  Between chunks the plain kernels leave the scaling to
        // scale_pass, which runs while the next chunk's MMA 1/2 are in flight.
        // SW state columns per round of a pass: 64 (both TMEM loads in flight
        // before one wait) in the plain kernels, 32 in the variants with the
        // norms or the extended features, which have fewer registers to spare
        constexpr int SW = (L2N || EXT) ? 32 : 64;
        // the plain kernels scale the state while MMA 1/2 run (scale_pass);
        // the heavier variants keep the single pass after MMA 3, whose
        // registers they can afford
        constexpr bool kSplitPass = !L2N && !EXT;
        auto ld_round = [&](int cb, uint32_t (&d)[SW]) {
            tmem_ld32(t_s + SW * cb, *reinterpret_cast<uint32_t(*)[32]>(&d[0]));
            if constexpr (SW == 64) tmem_ld32(t_s + SW * cb + 32, *reinterpret_cast<uint32_t(*)[32]>(&d[SW - 32]));
            tc_wait_ld();
        };
        auto st_round = [&](int cb, uint32_t (&d)[SW]) {
            tmem_st32(t_s + SW * cb, *reinterpret_cast<uint32_t(*)[32]>(&d[0]));
            if constexpr (SW == 64) tmem_st32(t_s + SW * cb + 32, *reinterpret_cast<uint32_t(*)[32]>(&d[SW - 32]));
        };
        auto scale_round = [&](const float *gam, int cb, uint32_t (&d)[SW]) {
#pragma unroll
            for (int e4 = 0; e4 < SW / 4; ++e4) {
                const float4 gm = *reinterpret_cast<const float4 *>(&gam[SW * cb + 4 * e4]);
                const float2 a = f2mul(make_float2(__uint_as_float(d[4 * e4]), __uint_as_float(d[4 * e4 + 1])),
                                       make_float2(gm.x, gm.y));
                const float2 b = f2mul(make_float2(__uint_as_float(d[4 * e4 + 2]), __uint_as_float(d[4 * e4 + 3])),
                                       make_float2(gm.z, gm.w));
                d[4 * e4] = __float_as_uint(a.x);
                d[4 * e4 + 1] = __float_as_uint(a.y);
                d[4 * e4 + 2] = __float_as_uint(b.x);
                d[4 * e4 + 3] = __float_as_uint(b.y);
            }
        };
        auto state_pass = [&](const float *gam_next, bool from_init, float *snap_out, bool last) {
#pragma unroll 1
            for (int cb = 0; cb < DK / SW; ++cb) {
                uint32_t d[SW];
                if (from_init) {
#pragma unroll
                    for (int e = 0; e < SW; ++e) {
                        const int i = SW * cb + e;
                        d[e] = __float_as_uint(identity ? (i == j ? 1.f : 0.f)
                                                        : (s_init ? s_init[(size_t)i * NC + j] : 0.f));
                    }
                } else {
                    ld_round(cb, d);
                    if (snap_out) {  // a state snapshot after this chunk
#pragma unroll
                        for (int e = 0; e < SW; ++e) snap_out[(size_t)(SW * cb + e) * NC + j] = __uint_as_float(d[e]);
                    }
                }
                if (!last) {
                    uint32_t pk[SW / 2];
#pragma unroll
                    for (int e = 0; e < SW / 2; ++e)
                        pk[e] = pack_bf16(__uint_as_float(d[2 * e]), __uint_as_float(d[2 * e + 1]));
                    if constexpr (SW == 64) tmem_st32(t_as + 32 * cb, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
                    else tmem_st16(t_as + 16 * cb, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                }
                if (gam_next) {
                    scale_round(gam_next, cb, d);
                    st_round(cb, d);
                } else if (last && s_out) {  // after the last chunk: the final state
#pragma unroll
                    for (int e = 0; e < SW; ++e) s_out[(size_t)(SW * cb + e) * NC + j] = __uint_as_float(d[e]);
                }
            }
            tc_wait_st();
            tc_fence_before();
        };
        // The fp32 state scaled in place by the chunk's exp(G_C) (gam), ahead
        // of the MMA 3 that accumulates into it; the TMEM stores are complete
        // on return.
        auto scale_pass = [&](const float *gam) {
#pragma unroll 1
            for (int cb = 0; cb < DK / SW; ++cb) {
                uint32_t d[SW];
                ld_round(cb, d);
                scale_round(gam, cb, d);
                st_round(cb, d);
            }
            tc_wait_st();
        };

        if (nchunks == 0) {
            if (s_out) {
#pragma unroll 4
                for (int i = 0; i < DK; ++i)
                    s_out[(size_t)i * NC + j] = identity ? (i == j ? 1.f : 0.f)
                                                         : (s_init ? s_init[(size_t)i * NC + j] : 0.f);
            }
        } else {
            bar_sync(BAR_FULL + 0, kBarCount);  // stage of chunk 0: its exp(G_C)
            if (ok) state_pass(sm.st[0].gam, true, nullptr, false);
        }
        // MMA operand descriptors of stage 0; stages are contiguous, so stage s
        // adds s * sizeof(Stage) / 16 to the start-address field (all of shared
        // memory is below 256 KB: the 14-bit field never carries)
        const uint64_t dsc_v0 = sdesc(smem_u32(sm.st[0].v), 128, 256);
        const uint64_t dsc_b00 = sdesc(smem_u32(sm.st[0].b0), 128, 256);
        const uint64_t dsc_b10 = sdesc(smem_u32(sm.st[0].b1), 128, DK * 16);
        const uint64_t dsc_b20 = sdesc(smem_u32(sm.st[0].b2), 128, 256);
        const uint64_t dsc_b30 = sdesc(smem_u32(sm.st[0].b3), 128, 256);
        const uint64_t dsc_au = sdesc(smem_u32(au), 128, 256);
        constexpr uint64_t kStageStep = sizeof(typename Lay::Stage) / 16;
        static_assert(sizeof(typename Lay::Stage) % 16 == 0, "stage stride");

        // Per chunk c:  [gate(c) -> io]  MMA 1/2 (c)  |  y(c-1) = gate (.) O
        //               U -> smem  MMA 3/4 (c)  |  y(c-1) -> global
        //               next stage; state pass
        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % kStages;
            const uint32_t d1_col = Lay::COL_D1 + 32 * (c & 1);
            if (OUT) cp_async_wait<0>();  // this thread's pieces of the gate tile of chunk c - 1
            bar_sync(bar_wg, 128);        // state-pass TMEM stores; gate tile; y(c - 2) stored
            if (OUT) load_gate(c);
            if (wwarp == 0 && ok) {  // U0^T and [-W | Qd] S^T: needs only the bf16 copy
                const uint32_t d1 = tbase + colb + d1_col;
                const uint64_t so = kStageStep * stg;
                if (elect_one_sync()) {
                    tc_fence_after();
                    if (use_v) tc_mma_ss(d1, dsc_v0 + so, dsc_b00 + so, ID_U0, 0);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)  // +256 bytes of K = +16 in the start field
                        tc_mma_ts(d1, tbase + colb + Lay::COL_AS + 8 * kk, dsc_b10 + so + 16 * kk, ID_WS,
                                  (use_v || kk > 0) ? 1u : 0u);
                    tc_commit(mb1);
                }
                __syncwarp();  // reconverge warp 0 before the aligned TMEM loads below
            }
            if (kSplitPass && c > 0 && ok) scale_pass(sm.st[stg].gam);  // S_{c-1} -> Diag(exp G_C) S_{c-1}
            if (c > 0) finish_chunk(c - 1);
            if (ok) ok = mbar_wait(mb1, c & 1);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {  // U^T row j -> bf16 A operand in shared memory
                uint32_t u[16];
                tmem_ld16_wait(t_d1 + 32 * (c & 1), u);
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    pk[e] = pack_bf16(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
                *reinterpret_cast<uint4 *>(at_bytes(au, kmaj(j, 0, 16))) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4 *>(at_bytes(au, kmaj(j, 8, 16))) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
            fence_async_smem();
            tc_fence_before();
            bar_sync(bar_wg, 128);
            if (wwarp == 0 && ok) {  // S^T += U^T Kb (into the state itself);  O^T += U^T P^T
                const uint64_t so = kStageStep * stg;
                if (elect_one_sync()) {
                    tc_fence_after();
                    tc_mma_ss(tbase + colb + Lay::COL_S, dsc_au, dsc_b20 + so, ID_UK, 1);
                    if (OUT) tc_mma_ss(tbase + colb + d1_col + 16, dsc_au, dsc_b30 + so, ID_UP, 1);
                    tc_commit(mb2);
                }
                __syncwarp();  // reconverge warp 0 before the aligned barrier below
            }
            const bool has_next = c + 1 < nchunks;
            if (OUT && c > 0) store_y(c - 1);
            if (has_next) bar_sync(BAR_FULL + (c + 1) % kStages, kBarCount);
            if (ok) ok = mbar_wait(mb2, c & 1);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            tc_fence_before();
            bar_arrive(BAR_EMPTY + stg, kBarCount);  // every reader of this stage is done
            if (ok) {
                state_pass(kSplitPass || !has_next ? nullptr : sm.st[(c + 1) % kStages].gam, false,
                           EXT ? snap.at(snap.pos0 + 16 * (c + 1)) : nullptr, !has_next);
            } else {
                tc_fence_before();
            }
        }
        if (nchunks > 0) {
            if (OUT) cp_async_wait<0>();
            bar_sync(bar_wg, 128);
            finish_chunk(nchunks - 1);
            if (OUT) {
                bar_sync(bar_wg, 128);
                store_y(nchunks - 1);
            }
        }
        if (active && !ok && lane == 0 && p.err) atomicOr(p.err, 1);
    } else if (kInterleave ? ((warp - 4 * NWG) & 1) == 0 : warp < 4 * NWG + 2) {
        // ------------------------------------------------------------ decay pair
        // In the plain kernels the first and third warp after the state warps
        // (their warp slots put them on two different SM sub-partitions, each
        // shared with a matrix warp); in the heavier variants, whose decay
        // work is longer, the first two (measured faster there).  Thread d
        // owns the key-channel pair (ip, ip + 1) on all 16 rows of a chunk; it
        // runs up to kRaw chunks ahead of the matrix pair.
        const int d = kInterleave ? 32 * ((warp - 4 * NWG) >> 1) + lane : tid - 128 * NWG;
        const int dw = d >> 5, ip = 2 * d;
        const bf16 *v = (const bf16 *)p.v, *beta = (const bf16 *)p.beta;
        typename Lay::Prep &pr = sm.pr;
        // beta of chunks c and c + 1 (threads d < 16), kept as raw bf16 bits so
        // that the load of chunk c + 2 is not waited for until it is stored
        unsigned short bq0 = 0, bq1 = 0;
        auto load_beta = [&](int c) -> unsigned short {
            const int rows = min(16, len - 16 * c);
            return d < rows ? reinterpret_cast<const unsigned short *>(beta)[(size_t)(t0 + 16 * c + d) * H + h]
                            : (unsigned short)0;
        };
        // V^T of chunk c -> its stage (MN-major A operand of MMA 1)
        auto issue_v = [&](int c) {
            if (USE_V) {
                typename Lay::Stage &Sv = sm.st[c % kStages];
                const int tc = t0 + 16 * c, rows = min(16, len - 16 * c);
                constexpr int PV = NC / 8;
#pragma unroll
                for (int x = d; x < 16 * PV; x += kPair) {
                    // token fastest: the 16-byte pieces of one warp fill whole
                    // core matrices (no bank conflicts) and pairs of them whole
                    // 32-byte sectors of v
                    const int r = x % 16, cc = x / 16;
                    const bool okr = r < rows;
                    const size_t off = ((size_t)(okr ? tc + r : t0) * H + h) * NC + cc * 8;
                    cp_async16(at_bytes(Sv.v, mnmaj(cc * 8, r, 16)), v + off, okr);
                }
            }
        };
        if (d < 16) {
            if (nchunks > 0) bq0 = load_beta(0);
            if (nchunks > 1) bq1 = load_beta(1);
        }
        bool tok = true;  // every raw tile arrived within the time bound

        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % kStages;
            typename Lay::Raw &Wk = sm.raw[c % kRaw];
            typename Lay::Stage &St = sm.st[stg];
            if (c >= kStages) bar_sync(BAR_EMPTY + stg, kBarCount);  // the stage is free again
            issue_v(c);
            cp_async_commit();
            unsigned short bq2 = 0;
            if (d < 16 && c + 2 < nchunks) bq2 = load_beta(c + 2);
            if (tok) tok = mbar_wait(smem_u32(&sm.mbar_raw[c % kRaw]), (c / kRaw) & 1);
            {   // rows past the end of the piece read as zero (decay 1, no write)
                const int rows = min(16, len - 16 * c);
                if (rows < 16) {
                    const int n = (16 - rows) * 2 * 8;  // 16-byte pieces per array
                    for (int x = d; x < 3 * n; x += kPair) {
                        const int a = x / n, y = x % n, r = rows + y / 16, hf = (y / 8) & 1, pc = y % 8;
                        unsigned char *base = a == 0 ? Wk.k : (a == 1 ? Wk.g : Wk.q);
                        *reinterpret_cast<uint4 *>(base + hf * 2048 + r * 128 + pc * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            if (d < 16) pr.beta[stg][d] = beta_in(__bfloat162float(__ushort_as_bfloat16(bq0)), flags);
            __syncwarp();
            bar_sync(BAR_DPAIR, kPair);             // the tiles (with cleared rows) are visible
            if (L2N) {  // row norms of k and q: the two warps cover all channels
                float sk[16], sq[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t *>(Wk.k + sw128(r, ip)));
                    sk[r] = kv.x * kv.x + kv.y * kv.y;
                    sq[r] = 0.f;
                    if (OUT) {
                        const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t *>(Wk.q + sw128(r, ip)));
                        sq[r] = qv.x * qv.x + qv.y * qv.y;
                    }
                }
                const float tk = warp_sum16_scatter(sk, lane);
                const float tq = OUT ? warp_sum16_scatter(sq, lane) : 0.f;
                if (!(lane & 1)) {
                    pr.nk[dw][row_of_lane(lane)] = tk;
                    pr.nq[dw][row_of_lane(lane)] = tq;
                }
                __syncwarp();
                bar_sync(BAR_DPAIR, kPair);
                if (d < 32) {  // 1/|k_r| and scale/|q_r|, once per row
                    const int r = d & 15;
                    float *dst = d < 16 ? pr.rk : pr.rq;
                    const float (*src)[16] = d < 16 ? pr.nk : pr.nq;
                    dst[r] = rsqrtf(src[0][r] + src[1][r] + 1e-6f) * (d < 16 ? 1.f : p.scale);
                }
                __syncwarp();
                bar_sync(BAR_DPAIR, kPair);
            }

            // exp(G_r) (inclusive prefix products of exp(g)), exp(G_C) and the
            // exclusive suffix products exp(G_C - G_r), in fp32
            float2 e[16], E[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float2 gg = unpack_bf16(*reinterpret_cast<const uint32_t *>(Wk.g + sw128(r, ip)));
                e[r] = make_float2(__expf(g_in(gg.x, flags)), __expf(g_in(gg.y, flags)));
            }
            {
                float2 acc = make_float2(1.f, 1.f);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    acc = f2mul(acc, e[r]);
                    E[r] = acc;
                }
            }
            const float2 El = E[15];
            const float2 invEl = make_float2(__frcp_rn(El.x), __frcp_rn(El.y));
            *reinterpret_cast<float2 *>(&St.gam[ip]) = El;
            uint32_t kb0[8], kb1[8];  // Kb^T rows ip, ip + 1 (token pairs)
            if constexpr (!L2N && !EXT) {
                // plain kernels: each tile column is loaded ahead of the in-place
                // stores (which would otherwise keep every load behind the
                // previous row's store); k last row first (the suffix products
                // run backwards), then q
                uint32_t kr[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) kr[r] = *reinterpret_cast<const uint32_t *>(Wk.k + sw128(r, ip));
                float2 F = make_float2(1.f, 1.f), kb_hi = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 15; r >= 0; --r) {
                    const float2 kv = unpack_bf16(kr[r]);
                    *reinterpret_cast<uint32_t *>(Wk.k + sw128(r, ip)) = pack_bf16(f2mul(kv, E[r]));
                    *reinterpret_cast<uint32_t *>(Wk.g + sw128(r, ip)) = pack_bf16(f2mul(kv, f2mul(F, invEl)));
                    const float2 kbv = f2mul(kv, F);
                    if (r & 1) {
                        kb_hi = kbv;
                    } else {
                        kb0[r >> 1] = pack_bf16(kbv.x, kb_hi.x);
                        kb1[r >> 1] = pack_bf16(kbv.y, kb_hi.y);
                    }
                    F = f2mul(F, e[r]);
                }
                if (OUT) {
                    uint32_t qr[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) qr[r] = *reinterpret_cast<const uint32_t *>(Wk.q + sw128(r, ip));
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        *reinterpret_cast<uint32_t *>(Wk.q + sw128(r, ip)) =
                            pack_bf16(f2mul(f2mul(unpack_bf16(qr[r]), make_float2(p.scale, p.scale)), E[r]));
                }
            } else {
                // the variants with the norms or the extended features (fewer
                // registers to spare): k and q row by row in one backward loop
                float2 F = make_float2(1.f, 1.f), kb_hi = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 15; r >= 0; --r) {
                    float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t *>(Wk.k + sw128(r, ip)));
                    float sc = p.scale;
                    if (L2N) {
                        const float rk = pr.rk[r];
                        kv = f2mul(kv, make_float2(rk, rk));
                        sc = pr.rq[r];
                    }
                    *reinterpret_cast<uint32_t *>(Wk.k + sw128(r, ip)) = pack_bf16(f2mul(kv, E[r]));
                    *reinterpret_cast<uint32_t *>(Wk.g + sw128(r, ip)) = pack_bf16(f2mul(kv, f2mul(F, invEl)));
                    const float2 kbv = f2mul(kv, F);
                    if (r & 1) {
                        kb_hi = kbv;
                    } else {
                        kb0[r >> 1] = pack_bf16(kbv.x, kb_hi.x);
                        kb1[r >> 1] = pack_bf16(kbv.y, kb_hi.y);
                    }
                    if (OUT) {
                        const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t *>(Wk.q + sw128(r, ip)));
                        *reinterpret_cast<uint32_t *>(Wk.q + sw128(r, ip)) =
                            pack_bf16(f2mul(f2mul(qv, make_float2(sc, sc)), E[r]));
                    }
                    F = f2mul(F, e[r]);
                }
            }
            *reinterpret_cast<uint4 *>(at_bytes(St.b2, kmaj(ip, 0, 16))) = make_uint4(kb0[0], kb0[1], kb0[2], kb0[3]);
            *reinterpret_cast<uint4 *>(at_bytes(St.b2, kmaj(ip, 8, 16))) = make_uint4(kb0[4], kb0[5], kb0[6], kb0[7]);
            *reinterpret_cast<uint4 *>(at_bytes(St.b2, kmaj(ip + 1, 0, 16))) = make_uint4(kb1[0], kb1[1], kb1[2], kb1[3]);
            *reinterpret_cast<uint4 *>(at_bytes(St.b2, kmaj(ip + 1, 8, 16))) = make_uint4(kb1[4], kb1[5], kb1[6], kb1[7]);
            // v of chunk c has landed; the stage's and the tile's generic writes
            // become visible to the tensor core and ordered before a TMA refill
            cp_async_wait<0>();
            fence_async_smem();
            bar_arrive(BAR_DEC + c % kRaw, kDecCount);
            bq0 = bq1;
            bq1 = bq2;
        }
        if (!tok && p.err) atomicOr(p.err, 2);
        // the stages of the last chunks come back before the CTA tears down
        for (int c = max(nchunks - kStages, 0); c < nchunks; ++c) bar_sync(BAR_EMPTY + c % kStages, kBarCount);
    } else {
        // ----------------------------------------------------------- matrix pair
        // The other two warps after the state warps: the Gram matrices, the
        // unit-lower solve, W, and the TMA loads of q, k, g (thread 0).
        const int m = kInterleave ? 32 * ((warp - 4 * NWG) >> 1) + lane : tid - 128 * NWG - kPair;
        const int mw = m >> 5;
        typename Lay::Prep &pr = sm.pr;
        auto issue_raw = [&](int c) {
            typename Lay::Raw &R = sm.raw[c % kRaw];
            const uint32_t mb = smem_u32(&sm.mbar_raw[c % kRaw]);
            const int tc = t0 + 16 * c;
            mbar_arrive_expect_tx(mb, (OUT ? 3u : 2u) * 16u * DK * 2u);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(smem_u32(R.k) + 2048 * hf, &maps.k, 64 * hf, h, tc, mb);
                tma_load_3d(smem_u32(R.g) + 2048 * hf, &maps.g, 64 * hf, h, tc, mb);
                if (OUT) tma_load_3d(smem_u32(R.q) + 2048 * hf, &maps.q, 64 * hf, h, tc, mb);
            }
        };
        if (m == 0)
            for (int c = 0; c < min(nchunks, kRaw); ++c) issue_raw(c);
        // rows 16-31 of every stage's [Tb^T | 0] operand stay zero
        for (int x = m; x < kStages * 32; x += kPair)
            reinterpret_cast<uint4 *>(at_bytes(sm.st[x / 32].b0, kmaj(16, 0, 16)))[x % 32] =
                make_uint4(0, 0, 0, 0);

        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % kStages;
            typename Lay::Raw &Wk = sm.raw[c % kRaw];
            typename Lay::Stage &St = sm.st[stg];
            const float *bet = pr.beta[stg];
            bar_sync(BAR_DEC + c % kRaw, kDecCount);  // Kd, Ki, Qd, Kb^T, exp(G_C), v of chunk c
            const unsigned char *Kd = Wk.k, *Ki = Wk.g, *Qd = Wk.q;

            // A = Kd Ki^T (warp 6) and P = Qd Ki^T (warp 7) on warp-level MMA
            if (mw == 0 || OUT) {
                const unsigned char *Aop = mw == 0 ? Kd : Qd;
                float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    uint32_t a[4], b[4];
                    ldsm4(a, Aop + sw128((lane & 7) + ((lane >> 3) & 1) * 8, 16 * kk + (lane >> 4) * 8));
                    ldsm4(b, Ki + sw128((lane & 7) + (lane >> 4) * 8, 16 * kk + ((lane >> 3) & 1) * 8));
                    mma16816(acc0, a, b[0], b[1]);
                    mma16816(acc1, a, b[2], b[3]);
                }
                const int r0 = lane >> 2, c0 = 2 * (lane & 3);
                if (mw == 0) {
                    // AT[s][r] = beta_r A[r][s] for s < r (the solve's column sweeps)
                    const float vals[8] = {acc0[0], acc0[1], acc0[2], acc0[3],
                                           acc1[0], acc1[1], acc1[2], acc1[3]};
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2) {
                        const int r = r0 + ((e2 & 2) ? 8 : 0);
                        const int sc = c0 + (e2 & 1) + ((e2 & 4) ? 8 : 0);
                        pr.AT[sc * kAT + r] = sc < r ? bet[r] * vals[e2] : 0.f;
                    }
                } else {
                    auto pv = [&](float x, int r, int sc) { return sc <= r ? x : 0.f; };
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b3, kmaj(r0, c0, 16))) =
                        pack_bf16(pv(acc0[0], r0, c0), pv(acc0[1], r0, c0 + 1));
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b3, kmaj(r0 + 8, c0, 16))) =
                        pack_bf16(pv(acc0[2], r0 + 8, c0), pv(acc0[3], r0 + 8, c0 + 1));
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b3, kmaj(r0, c0 + 8, 16))) =
                        pack_bf16(pv(acc1[0], r0, c0 + 8), pv(acc1[1], r0, c0 + 9));
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b3, kmaj(r0 + 8, c0 + 8, 16))) =
                        pack_bf16(pv(acc1[2], r0 + 8, c0 + 8), pv(acc1[3], r0 + 8, c0 + 9));
                }
            }
            __syncwarp();
            bar_sync(BAR_MPAIR, kPair);             // AT and P are written

            // Tb = (I + Diag(beta) A)^-1 Diag(beta): lane j < 16 of warp 6 owns
            // column j, and after row r is final it is pushed into every later
            // row.  Meanwhile warp 7 copies Qd into rows 16-31 of [-W | Qd].
            if (mw == 0) {
                if (lane < 16) {
                    const int jj = lane;
                    float col[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) col[r] = (r == jj) ? 1.f : 0.f;
#pragma unroll
                    for (int r = 0; r < 15; ++r) {
                        float at[16];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(&pr.AT[r * kAT + 4 * q4]);
                            at[4 * q4 + 0] = a4.x; at[4 * q4 + 1] = a4.y;
                            at[4 * q4 + 2] = a4.z; at[4 * q4 + 3] = a4.w;
                        }
#pragma unroll
                        for (int r2 = r + 1; r2 < 16; ++r2) col[r2] = fmaf(-at[r2], col[r], col[r2]);
                    }
                    const float bj = bet[jj];
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        *at_bytes(St.b0, kmaj(r, jj, 16)) = __float2bfloat16_rn(col[r] * bj);
                }
            } else if (OUT) {
#pragma unroll
                for (int it = 0; it < DK / 16; ++it) {
                    const int x = lane + 32 * it;
                    const int r = x & 15, kc = x >> 4;
                    *reinterpret_cast<uint4 *>(at_bytes(St.b1, kmaj(16 + r, 8 * kc, DK))) =
                        *reinterpret_cast<const uint4 *>(Qd + sw128(r, 8 * kc));
                }
            }
            __syncwarp();
            bar_sync(BAR_MPAIR, kPair);             // Tb is written

            // W = Tb Kd -> rows 0-15 of the [-W | Qd] operand hold -W; warp mw
            // covers key channels [DK/2 mw, DK/2 (mw + 1))
            {
                uint32_t a[4];
                ldsm4(a, at_bytes(St.b0, kmaj((lane & 7) + ((lane >> 3) & 1) * 8, (lane >> 4) * 8, 16)));
#pragma unroll
                for (int np = mw * (DK / 32); np < (mw + 1) * (DK / 32); ++np) {
                    const int n0 = 16 * np;
                    uint32_t b[4];
                    ldsm4t(b, Kd + sw128((lane & 7) + ((lane >> 3) & 1) * 8, n0 + (lane >> 4) * 8));
                    float w0[4] = {0.f, 0.f, 0.f, 0.f}, w1[4] = {0.f, 0.f, 0.f, 0.f};
                    mma16816(w0, a, b[0], b[1]);
                    mma16816(w1, a, b[2], b[3]);
                    const int r = lane >> 2, cc = n0 + 2 * (lane & 3);
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b1, kmaj(r, cc, DK))) = pack_bf16(-w0[0], -w0[1]);
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b1, kmaj(r + 8, cc, DK))) = pack_bf16(-w0[2], -w0[3]);
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b1, kmaj(r, cc + 8, DK))) = pack_bf16(-w1[0], -w1[1]);
                    *reinterpret_cast<uint32_t *>(at_bytes(St.b1, kmaj(r + 8, cc + 8, DK))) = pack_bf16(-w1[2], -w1[3]);
                }
            }
            // the stage's generic writes become visible to the tensor core; the
            // raw tile is no longer read by either pair: refill it
            fence_async_smem();
            __syncwarp();
            bar_sync(BAR_MPAIR, kPair);
            if (m == 0 && c + kRaw < nchunks) issue_raw(c + kRaw);
            bar_arrive(BAR_FULL + stg, kBarCount);
        }
    }

    // ---- tear-down: every TMEM access of the CTA is complete
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemCols)
                     : "memory");
}

// The summary pass: one CTA per (piece, head), one SM each.  State warpgroup
// 0 runs the piece from zero (or from the sequence's initial state for its
// first piece) into S_zero, warpgroup 1 runs it from the identity without v
// into the transition M; both share one preparation of every chunk.  A part
// the scan does not need (both maps of a sequence's last piece, M of its
// first) is skipped unless every piece's map is asked for.  The same holds
// for sub-pieces, piece by piece of the output pass.
template <int DK, bool L2N, bool EXT>
__global__ void __launch_bounds__(kThreadsOf<2>, 1)
    summary_kernel(PrefillParams p, const __grid_constant__ TmaMaps maps) {
    extern __shared__ __align__(128) unsigned char smem[];
    // (piece, head) pairs with the head fastest: co-resident CTAs cover all
    // heads of a few pieces, spreading their rows over every memory channel
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    // with sub-pieces, j counts sub-pieces and `sub` of them make one piece of
    // the output pass; a (sub-)piece is summarised when the output piece it
    // lies in has a successor, its transition too unless it starts the
    // sequence (the fold composes the sub-piece maps of each piece)
    const int sub = p.sub > 1 ? p.sub : 1;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    const bool needed = j / sub < (np + sub - 1) / sub - 1;
    const bool want_s = p.summarize_all || needed;
    const bool want_m = p.summarize_all || (needed && j > 0);
    if (!want_s && !want_m) return;
    const size_t ph = (size_t)pi * p.H + h;
    const float *init = (j == 0 && p.initial_state)
                            ? p.initial_state + ((size_t)n * p.H + h) * DK * NC
                            : nullptr;
    run_piece<DK, false, true, L2N, EXT, 2>(p, maps, pc.y, pc.z, h, init, false,
                                       want_s ? p.Szero + ph * DK * NC : nullptr, smem, Snap(),
                                       want_m ? p.M + ph * DK * DK : nullptr, want_s, want_m);
}

template <int DK, bool L2N, bool EXT>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM) output_kernel(PrefillParams p, const __grid_constant__ TmaMaps maps) {
    extern __shared__ __align__(128) unsigned char smem[];
    // (piece, head) pairs with the head fastest: co-resident CTAs cover all
    // heads of a few pieces, spreading their rows over every memory channel
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    const size_t nh = (size_t)n * p.H + h;
    const float *init = (np == 1) ? (p.initial_state ? p.initial_state + nh * DK * NC : nullptr)
                                  : p.Sin + ((size_t)pi * p.H + h) * DK * NC;
    float *fin = (j == np - 1 && p.final_state) ? p.final_state + nh * DK * NC : nullptr;
    run_piece<DK, true, true, L2N, EXT>(p, maps, pc.y, pc.z, h, init, false, fin, smem,
                                        EXT ? make_snap(p, n, h, pc.y, (size_t)DK * NC) : Snap());
}

}  // namespace tc5

// dk = dv = 128 only (one state column per TMEM lane; the transition part has
// dk columns too).
namespace {
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); null when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// [T][H][128] bf16 as a 3-D tensor (channel, head, token); box 64 x 1 x 16.
bool encode_rows(CUtensorMap *m, const void *base, int T, int H) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {256, (cuuint64_t)H * 256};
    const cuuint32_t box[3] = {64, 1, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool L2N, bool EXT>
cudaError_t launch_tc5(const PrefillParams &p, bool summaries, cudaStream_t st) {
    const size_t sm = tc5::Layout<128>::bytes;
    const size_t sm2 = tc5::Layout<128, 2>::bytes;
    cudaError_t e;
    tc5::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (p.total_tokens > 0 &&
        (!encode_rows(&maps.q, p.q, p.total_tokens, p.H) || !encode_rows(&maps.k, p.k, p.total_tokens, p.H) ||
         !encode_rows(&maps.g, p.g, p.total_tokens, p.H)))
        return cudaErrorInvalidValue;
    if (summaries) {
        e = cudaFuncSetAttribute(tc5::summary_kernel<128, L2N, EXT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
        if (e != cudaSuccess) return e;
        tc5::summary_kernel<128, L2N, EXT><<<dim3((unsigned)(p.P_max * p.H)), tc5::kThreadsOf<2>, sm2, st>>>(
            p, maps);
        return cudaGetLastError();
    }
    e = cudaFuncSetAttribute(tc5::output_kernel<128, L2N, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm);
    if (e != cudaSuccess) return e;
    tc5::output_kernel<128, L2N, EXT><<<dim3((unsigned)(p.P_max * p.H)), tc5::kThreads, sm, st>>>(p, maps);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_prefill_tc5(const PrefillParams &p, bool summaries, cudaStream_t st) {
    const bool l2 = p.flags & FLAG_L2NORM;
    const bool ext = (p.flags & ~FLAG_L2NORM) || p.snap_tokens > 0;
    if (ext) return l2 ? launch_tc5<true, true>(p, summaries, st) : launch_tc5<false, true>(p, summaries, st);
    return l2 ? launch_tc5<true, false>(p, summaries, st) : launch_tc5<false, false>(p, summaries, st);
}

}  // namespace kda
