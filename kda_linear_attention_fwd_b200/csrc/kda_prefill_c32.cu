// KDA prefill for bf16, dk = dv = 128, with the state carried across
// 32-token chunks: every dense product of the chunk on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Decay ratios are only ever taken inside a 16-token tile, the length that
// keeps them within BF16 range at the decay floor (prism.simon-ai.net,
// "从架构创新出发：K3的MoE与混合注意力设计", section "数值稳定性与 Co-Design：BF16
// 约束下的衰减控制策略"); the state is handed on once per two tiles, so the
// serial part of the work -- one pass over the fp32 state and two tensor-core
// round trips -- happens half as often as with 16-token chunks.  The split
// into parallel per-chunk preparation and a sequential state pass follows the
// affta.cn K3 explainer, section "FlashKDA ，让线性计算也能沾上并行的光"; the
// token pipeline (forget, delta write, read, output gate) its section
// "第一关：KDA 解决算得动".
//
// Per chunk of 32 tokens (sub-tiles c = 0, 1 of 16 rows; within tile c,
// E_c[r] = prod_{u<=r} exp(g_u), F_c[r] = prod_{u>r} exp(g_u), gamma_c =
// E_c[15], products over the tile's own rows):
//   Kd_c = k E_c, Ki_c = k / E_c, Kb_c = k F_c, Qd_c = scale q E_c
//   A = [[sl(Kd_0 Ki_0^T), 0], [Kd_1 Kb_0^T, sl(Kd_1 Ki_1^T)]]   (strictly lower)
//   P = [[tl(Qd_0 Ki_0^T), 0], [Qd_1 Kb_0^T, tl(Qd_1 Ki_1^T)]]   (lower, diagonal in)
//   T~ = (I + Diag(beta) A)^-1 Diag(beta)           (fp32 forward substitution)
//   K~ = [Kd_0; gamma_0 Kd_1],  Q~ = [Qd_0; gamma_0 Qd_1],  Kbar = [gamma_1 Kb_0; Kb_1]
//   W = T~ K~,  U = T~ V - W S,  O = Q~ S + P U,  S <- gamma_0 gamma_1 S + Kbar^T U
// (the same algebra as 16-token chunks, with the cross-tile terms written
// out; every factor is at most 1 except Ki, which stays within one tile).
//
// Tensor-core products per chunk, all tcgen05.mma kind::f16 (bf16 in, fp32
// accumulate), issued by one elected thread, completion through
// tcgen05.commit -> mbarrier:
//   AP  D[64 x 48]  = [Qd_0; Qd_1; Kd_0; Kd_1] [Ki_0; Ki_1; Kb_0]^T    (M=64, K=128)
//       -> every block of P and A at once; operands are the TMA tiles
//          themselves (K-major, 128-byte swizzle), rewritten in place
//   W   D[128 x 32] = Kd_0^T T~[:, 0:16]^T,  Kd_1^T T~[:, 16:32]^T      (M=128, K=16)
//       -> W^T = X + Diag(gamma_0) Y, the k tile read MN-major in place
//   1   D1         = V^T [T~^T | 0]                                 (M=128, N=64, K=32)
//   2   D1        += S^T [-W^T | Q~^T]     -> D1 = [U^T | (Q~ S)^T]  (K=128, A = S^T in TMEM)
//   3   S^T       += U^T Kbar                                       (N=128, K=32)
//   4   D1[32:64] += U^T P^T               -> O^T                   (N=32, K=32)
//
// One CTA (512 threads, one per SM) runs one piece of one head:
//   warps 0-7  state team: the fp32 S^T (TMEM lane j = state column j) and
//              MMAs 1-4; output pass: one chain, warps w and w+4 share lane
//              quarter w and split the state columns; summary pass: warps
//              0-3 run the piece from zero (or its initial state), warps 4-7
//              from the identity without v (the transition)
//   warps 8-11 decay team: thread (tile, key-channel pair): exp(g), the
//              prefix / suffix products and every scaled copy above, Q~ and
//              Kbar straight into the operand layouts, beta
//   warps 12-15 matrix team: MMA AP and its read-out (P into its operand,
//              beta A for the solve), the 32 x 32 unit-lower solve (one warp,
//              one column per lane, fp32), MMA W and its read-out (-W into
//              its operand), TMA refills of q, k, g
// Hand-offs: decay -> matrix (named barrier DEC, per tile buffer), decay ->
// state (mbarrier mb_gam: the chunk's gamma, all the next state pass needs),
// matrix -> state (FULL: every operand of the chunk), state -> decay (EMPTY:
// the update MMAs that read a stage have completed, so it may be refilled).
// Every wait on an mbarrier is bounded (2 s); a wait that gives up sets an
// error bit in the workspace header and the CTA drains through its barriers
// without further tensor work.
#include "kda_common.cuh"
#include "kda_prefill.cuh"
#include "kda_sm100.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

namespace kda {
namespace c32 {

using namespace sm100;

constexpr int kC = 32;           // tokens per state step
constexpr int kD = 128;          // dk = dv
constexpr int kThreads = 512;
// one chunk of raw tiles: per 64-channel half, q (32 rows) | k (32) | g (32)
// | Kb_0 (16), 128 bytes a row, 128-byte swizzle, every tile 1024-aligned
constexpr int kHalf = 14336;
constexpr int OFF_Q = 0, OFF_K = 4096, OFF_G = 8192, OFF_KB = 12288;
constexpr int kRawBytes = 2 * kHalf;

// Pipeline depths: NS prepared stages (chunk c -> stage c % NS) and NR chunks
// of q, k, g tiles (chunk c -> raw[c % NR]).  The output pass keeps three
// stages so that the preparation runs further ahead of the state chain; the
// summary pass, whose stage data is smaller but which keeps a second state
// copy in shared memory, keeps two stages and three tile buffers.
template <bool OUT> struct Pipe {
    static constexpr int NS = OUT ? 3 : 2;
    static constexpr int NR = OUT ? 2 : 3;
    // named barriers (0 is __syncthreads)
    static constexpr int FULL = 1;             // NS: matrix team arrives (128), state team waits (256)
    static constexpr int EMPTY = FULL + NS;    // NS: state team arrives (256), decay team waits (128)
    static constexpr int DEC = EMPTY + NS;     // NR: decay team arrives (128), matrix team waits (128)
    static constexpr int STATE = DEC + NR;     // 3: output pass: the state team (256), its U half
                                               //    (warps 0-3) and its O half (warps 4-7); summary:
                                               //    one per chain (128)
    static constexpr int DECAY = STATE + 3;    // decay team only
    static constexpr int MAT = DECAY + 1;      // matrix team only
    static_assert(MAT <= 15, "named barrier ids");
};
constexpr int kFullCount = 384, kEmptyCount = 384, kDecCount = 256;

// Byte offset of element (row r, channel ch) in a chunk of raw tiles, tile at
// offset `tile` of each half.
KDA_DEVICE uint32_t rsw(int tile, int r, int ch) {
    return (uint32_t)((ch >> 6) * kHalf + tile + r * 128 + ((((ch & 63) >> 3) ^ (r & 7)) << 4) + ((ch & 7) << 1));
}

struct alignas(1024) Stage {
    unsigned char v[8192];    // V tile, TMA (2 halves x 32 rows x 128 B, swizzled): A of MMA 1, MN-major
    unsigned char b1[16384];  // [-W | Q~] as B of MMA 2: MN-major [K=128][N=64], no swizzle
    unsigned char b0[4096];   // [T~ ; 0] as B of MMA 1 / W: K-major [64][32]
    unsigned char b2[8192];   // Kbar^T as B of MMA 3: K-major [128 channels][32 tokens]
    unsigned char b3[2048];   // P as B of MMA 4: K-major [32][32]
    float gam[kD];            // gamma_0 gamma_1 per key channel
    float beta[kC];
};

template <bool OUT>
struct Smem {
    alignas(1024) unsigned char raw[Pipe<OUT>::NR][kRawBytes];
    Stage st[Pipe<OUT>::NS];
    alignas(16) unsigned char au[OUT ? 1 : 2][8192];         // U^T as A of MMA 3/4: K-major [128][32]
    alignas(16) unsigned char mbf[OUT ? 16 : 32768];         // summary: bf16 transition, K-major [128][128]
    alignas(128) unsigned char io[OUT ? 2 : 1][OUT ? 8192 : 16];  // gate tile in, y tile out ([32][128] bf16)
    alignas(16) float AT[kC * kC];                           // AT[s][r] = beta_r A[r][s]
    alignas(16) float Td[2][16 * 16];                        // fp32 diagonal blocks of T
    alignas(16) float Zx[16 * 16];                           // N10 T00
    alignas(16) float gexch[2][kD];                          // gamma of each tile (decay team)
    alignas(16) float gam0[Pipe<OUT>::NS][kD];               // gamma_0 per chunk (W read-out)
    // mb_gam[s]: the 128 decay threads arrive once gamma of the stage's chunk is
    // written (all the state pass needs); the state team waits on it
    alignas(8) unsigned long long mb_raw[Pipe<OUT>::NR], mb_ap[Pipe<OUT>::NS], mb_gam[Pipe<OUT>::NS], mb_w,
        mb1[2], mb2[2];
    uint32_t tmem_base;
};
template <bool OUT> constexpr size_t kSmemBytes = sizeof(Smem<OUT>) + 1024;
static_assert(kSmemBytes<true> <= 232448 && kSmemBytes<false> <= 232448, "shared memory per CTA");
constexpr int kPrefetch = 6;   // chunks ahead whose tiles are pulled into L2

// TMEM columns (512 allocated)
template <bool OUT> struct Cols;
// AP: one 64-column buffer per stage (chunk c -> c % NS); the W product of
// a chunk reuses its AP buffer once the Gram blocks have been read out.
template <> struct Cols<true> {
    static constexpr uint32_t S = 0, BF = 128, D1 = 192, AP = 320;  // D1: 2 x 64, AP: 3 x 64
};
template <> struct Cols<false> {
    // chain 0 (zero start): S, its bf16 copy, D1; chain 1 (transition): S2, D1b
    // (its bf16 copy lives in shared memory)
    static constexpr uint32_t S = 0, BF = 128, D1 = 192, D1b = 224, S2 = 256, AP = 384;
};

// TMA descriptors of q, k, g as [T][H][128] bf16 (3-D: channel, head,
// token), box 64 x 1 x 32 with the 128-byte swizzle.  v and the gate arrive
// by cp.async and y leaves by plain stores: the SM's TMA unit serves the
// three tiles of every chunk and their L2 prefetches only.
struct Maps {
    CUtensorMap q, k, g;
};

KDA_DEVICE void prefetch_l2(const void *p) { asm volatile("prefetch.L2 [%0];" ::"l"(p)); }

KDA_DEVICE bool all_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

// Runs tokens [t0, t0 + len) of head h.  Output pass (OUT): the state starts
// at s_init (or zero) and ends in s_out (if given); y is written.  Summary
// pass: chain 0 from s_init (or zero) into s_out, chain 1 from the identity
// without v into m_out; a chain whose output is not wanted (null) does no
// tensor work but keeps every hand-off.
template <bool OUT>
__device__ void run_piece(const PrefillParams &p, const Maps &maps, int t0, int len, int h,
                          const float *s_init, float *s_out, float *m_out, unsigned char *smem_raw) {
    using L = Cols<OUT>;
    using PP = Pipe<OUT>;
    Smem<OUT> &sm = *reinterpret_cast<Smem<OUT> *>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    const int nchunks = (len + kC - 1) / kC;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm.tmem_base)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 32) {
        for (int i = 0; i < Pipe<OUT>::NR; ++i) mbar_init(smem_u32(&sm.mb_raw[i]), 1);
        for (int i = 0; i < Pipe<OUT>::NS; ++i) {
            mbar_init(smem_u32(&sm.mb_ap[i]), 1);
            mbar_init(smem_u32(&sm.mb_gam[i]), 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.mb1[i]), 1);
            mbar_init(smem_u32(&sm.mb2[i]), 1);
        }
        mbar_init(smem_u32(&sm.mb_w), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp < 8) {
        // =========================================================== state team
        const int wq = warp & 3;                       // TMEM lane quarter
        const int j = tid & 127;                       // state column = TMEM lane
        const int hf = tid >> 7;                       // output: column half; summary: chain
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int chain = OUT ? 0 : hf;
        const bool use_v = chain == 0;
        const bool active = OUT ? true : (chain == 0 ? s_out != nullptr : m_out != nullptr);
        const int bar_team = OUT ? PP::STATE : PP::STATE + chain;
        const int team_n = OUT ? 256 : 128;
        // columns of S^T this thread keeps: output 64 (one half), summary all 128
        constexpr int NCOL = OUT ? 64 : 128;
        const int c0 = OUT ? 64 * hf : 0;
        const uint32_t col_s = chain == 0 ? L::S : Cols<false>::S2;  // S^T of this chain
        const uint32_t t_s = tbase + lane_off + col_s + c0;
        const uint32_t t_bf = tbase + lane_off + L::BF + c0 / 2;
        const float *init = chain == 0 ? s_init : nullptr;  // chain 1 starts at the identity
        float *fin = chain == 0 ? s_out : m_out;
        const uint32_t mb1 = smem_u32(&sm.mb1[chain]), mb2 = smem_u32(&sm.mb2[chain]);
        unsigned char *au = sm.au[OUT ? 0 : chain];
        const bool issuer = (warp & 3) == 0;           // warp 0 (and warp 4 for chain 1)
        const bool issue_team = OUT ? warp == 0 : issuer;
        bool ok = active;
        const bf16 *gate = (const bf16 *)p.gate;
        bf16 *out = (bf16 *)p.out;

        // MMA operand descriptors (stage 0; stage s adds s * sizeof(Stage))
        constexpr uint32_t kStageStep = sizeof(Stage) >> 4;
        const uint64_t dsc_v = sdesc_sw128(smem_u32(sm.st[0].v), 4096, 1024);
        const uint64_t dsc_b0 = sdesc(smem_u32(sm.st[0].b0), 128, 512);
        const uint64_t dsc_b1 = sdesc(smem_u32(sm.st[0].b1), 128, 2048);
        const uint64_t dsc_b2 = sdesc(smem_u32(sm.st[0].b2), 128, 512);
        const uint64_t dsc_b3 = sdesc(smem_u32(sm.st[0].b3), 128, 512);
        const uint64_t dsc_au = sdesc(smem_u32(au), 128, 512);
        const uint64_t dsc_mbf = sdesc(smem_u32(sm.mbf), 128, 2048);
        constexpr int N1 = OUT ? 64 : 32;
        constexpr uint32_t ID_1 = idesc_bf16(128, N1, 1, 0);   // V^T (MN-major) x [T~ | 0]
        constexpr uint32_t ID_2 = idesc_bf16(128, N1, 0, 1);   // S^T x [-W | Q~] (MN-major B)
        constexpr uint32_t ID_3 = idesc_bf16(128, 128, 0, 0);  // U^T x Kbar
        constexpr uint32_t ID_4 = idesc_bf16(128, 32, 0, 0);   // U^T x P^T
        auto d1_addr = [&](int c) -> uint32_t {
            return OUT ? L::D1 + 64 * (c & 1) : (chain == 0 ? Cols<false>::D1 : Cols<false>::D1b);
        };

        // One pass over this thread's state columns: the bf16 copy (A of the
        // next MMA 2: TMEM for chain 0, shared memory for the transition) and,
        // when a next chunk exists, the state pre-scaled by its gamma so that
        // its MMA 3 accumulates into it; after the last chunk, the state out.
        auto state_pass = [&](bool from_init, const float *gam_next) {
#pragma unroll 1
            for (int cb = 0; cb < NCOL; cb += 64) {
                uint32_t d[64];
                if (from_init) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const int i = c0 + cb + e;
                        d[e] = __float_as_uint(chain == 1 ? (i == j ? 1.f : 0.f)
                                                          : (init ? init[(size_t)i * kD + j] : 0.f));
                    }
                } else {
                    uint32_t(&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&d[0]);
                    uint32_t(&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&d[32]);
                    tmem_ld32(t_s + cb, lo);
                    tmem_ld32(t_s + cb + 32, hi);
                    tc_wait_ld();
                }
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(__uint_as_float(d[2 * e]), __uint_as_float(d[2 * e + 1]));
                if (chain == 0) {
                    tmem_st32(t_bf + cb / 2, pk);
                } else {  // K-major [128 j][128 i]: row j, 8 channels per 16 bytes
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8)
                        *reinterpret_cast<uint4 *>(sm.mbf + kmaj(j, cb + 8 * q8, 128)) =
                            make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
                }
                if (gam_next) {
#pragma unroll
                    for (int e4 = 0; e4 < 16; ++e4) {
                        const float4 gm = *reinterpret_cast<const float4 *>(&gam_next[c0 + cb + 4 * e4]);
                        const float2 a = f2mul(make_float2(__uint_as_float(d[4 * e4]), __uint_as_float(d[4 * e4 + 1])),
                                               make_float2(gm.x, gm.y));
                        const float2 b = f2mul(make_float2(__uint_as_float(d[4 * e4 + 2]), __uint_as_float(d[4 * e4 + 3])),
                                               make_float2(gm.z, gm.w));
                        d[4 * e4] = __float_as_uint(a.x);
                        d[4 * e4 + 1] = __float_as_uint(a.y);
                        d[4 * e4 + 2] = __float_as_uint(b.x);
                        d[4 * e4 + 3] = __float_as_uint(b.y);
                    }
                    tmem_st32(t_s + cb, *reinterpret_cast<uint32_t(*)[32]>(&d[0]));
                    tmem_st32(t_s + cb + 32, *reinterpret_cast<uint32_t(*)[32]>(&d[32]));
                } else if (fin) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) fin[(size_t)(c0 + cb + e) * kD + j] = __uint_as_float(d[e]);
                }
            }
            if (chain == 1) fence_async_smem();
            tc_wait_st();
            tc_fence_before();
        };

        // Output pass: warps 4-7 (the O half) produce y of the previous chunk
        // while warps 0-3 (the U half) turn this chunk's U into the operand of
        // MMA 3/4, so the epilogue stays off the state chain.
        // Gate tile of chunk c -> io[c & 1] by cp.async: O-half thread j moves
        // the 16-byte pieces j + 128 i (row x / 16, piece x % 16), the same
        // pieces it stores as y, so a buffer is refilled right after its y left
        // without a barrier.  One commit group per chunk (empty when there is
        // nothing to load), so that wait_group 1 leaves exactly the newest one
        // in flight.
        auto issue_gate = [&](int c) {
            if (gate && c < nchunks) {
                const int rows = min(kC, len - kC * c);
                unsigned char *tile = sm.io[c & 1];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int x = j + 128 * i, r = x >> 4, cc = x & 15;
                    const bool okr = r < rows;
                    cp_async16(tile + r * 256 + cc * 16,
                               gate + ((size_t)(t0 + kC * c + (okr ? r : 0)) * H + h) * kD + cc * 8, okr);
                }
            }
            cp_async_commit();
        };
        // L2 prefetch of the gate rows of chunk c (one 128-byte line per thread)
        auto prefetch_gate = [&](int c) {
            if (gate && c < nchunks && j < 64) {
                const int r = j >> 1;
                if (kC * c + r < len) prefetch_l2(gate + ((size_t)(t0 + kC * c + r) * H + h) * kD + (j & 1) * 64);
            }
        };
        // y = gate (.) O of chunk c (O half): column j, all 32 rows, in place in
        // the gate tile; then the tile's rows to global and the buffer refilled
        // with the gate of chunk c + 2
        auto epilogue = [&](int c) {
            const int rows = min(kC, len - kC * c);
            unsigned char *tile = sm.io[c & 1];
            cp_async_wait<1>();  // the gate of chunk c (chunk c + 1's may still be in flight)
            bar_sync(PP::STATE + 2, 128);
            if (ok) {
                uint32_t o[32];
                tmem_ld32(tbase + lane_off + d1_addr(c) + 32, o);
                tc_wait_ld();
                bf16 *tl = reinterpret_cast<bf16 *>(tile);
#pragma unroll
                for (int t = 0; t < kC; ++t) {
                    const float gv = gate ? __bfloat162float(tl[t * kD + j]) : 1.f;
                    tl[t * kD + j] = __float2bfloat16_rn(gv * __uint_as_float(o[t]));
                }
            }
            tc_fence_before();
            bar_sync(PP::STATE + 2, 128);
            if (ok) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int x = j + 128 * i, r = x >> 4, cc = x & 15;
                    if (r < rows)
                        *reinterpret_cast<uint4 *>(out + ((size_t)(t0 + kC * c + r) * H + h) * kD + cc * 8) =
                            *reinterpret_cast<const uint4 *>(tile + r * 256 + cc * 16);
                }
            }
            issue_gate(c + 2);
            prefetch_gate(c + 6);
        };
        // U^T of chunk c (tokens u0 .. u0 + 31 of this thread's column) -> bf16
        // A operand of MMA 3/4
        auto u_readout = [&](int c) {
            if (ok) ok = mbar_wait(mb1, c & 1);
            ok = all_ok(ok);
            tc_fence_after();
            if (ok) {
                uint32_t u[32];
                tmem_ld32(tbase + lane_off + d1_addr(c), u);
                tc_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(au + kmaj(j, 8 * q8, kC)) =
                        make_uint4(pack_bf16(__uint_as_float(u[8 * q8 + 0]), __uint_as_float(u[8 * q8 + 1])),
                                   pack_bf16(__uint_as_float(u[8 * q8 + 2]), __uint_as_float(u[8 * q8 + 3])),
                                   pack_bf16(__uint_as_float(u[8 * q8 + 4]), __uint_as_float(u[8 * q8 + 5])),
                                   pack_bf16(__uint_as_float(u[8 * q8 + 6]), __uint_as_float(u[8 * q8 + 7])));
            }
            fence_async_smem();
            tc_fence_before();
        };
        auto wait_gamma = [&](int c) {  // gamma of chunk c is in its stage
            if (ok) ok = mbar_wait(smem_u32(&sm.mb_gam[c % PP::NS]), (c / PP::NS) & 1);
            ok = all_ok(ok);
        };

        if (OUT && hf == 1) {
            issue_gate(0);
            issue_gate(1);
            for (int c = 0; c < 6; ++c) prefetch_gate(c);
        }
        if (nchunks == 0) {
            if (fin) {
                for (int i = c0; i < c0 + NCOL; ++i)
                    fin[(size_t)i * kD + j] = chain == 1 ? (i == j ? 1.f : 0.f) : (init ? init[(size_t)i * kD + j] : 0.f);
            }
        } else {
            wait_gamma(0);
            if (active && ok) state_pass(true, sm.st[0].gam);
            tc_fence_before();
            bar_sync(bar_team, team_n);
        }

        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % PP::NS;
            const uint64_t so = (uint64_t)kStageStep * stg;
            const uint32_t d1 = tbase + d1_addr(c);
            bar_sync(PP::FULL + stg, kFullCount);  // every operand of chunk c is in its stage
            // ---- MMA 1 and 2: U^T and (Q~ S)^T, from the bf16 copy of S^T
            if (issue_team && ok) {
                if (elect_one_sync()) {
                    tc_fence_after();
                    if (use_v) {
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)  // 16 tokens = 2048 bytes of the V tile
                            tc_mma_ss(d1, dsc_v + so + 128 * kk, dsc_b0 + so + 16 * kk, ID_1, kk > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // 16 channels = 256 bytes of [-W | Q~]
                        if (chain == 0)
                            tc_mma_ts(d1, tbase + L::BF + 8 * kk, dsc_b1 + so + 16 * kk, ID_2,
                                      (use_v || kk > 0) ? 1u : 0u);
                        else
                            tc_mma_ss(d1, dsc_mbf + 16 * kk, dsc_b1 + so + 16 * kk, ID_2, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(mb1);
                }
                __syncwarp();
            }
            const bool issue34 = OUT ? (hf == 0) : true;  // threads that feed MMA 3/4
            if (OUT && hf == 1) {
                if (c > 0) epilogue(c - 1);  // the previous chunk's output, while MMA 1/2 run
            } else {
                u_readout(c);
                bar_sync(OUT ? PP::STATE + 1 : bar_team, 128);  // the U half (output) or the chain
            }
            // ---- MMA 3 (state update) and 4 (P U into O)
            if (issue34 && issue_team && ok) {
                if (elect_one_sync()) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_ss(tbase + col_s, dsc_au + 16 * kk, dsc_b2 + so + 16 * kk, ID_3, 1u);
                    if (OUT) {
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
                            tc_mma_ss(d1 + 32, dsc_au + 16 * kk, dsc_b3 + so + 16 * kk, ID_4, 1u);
                    }
                    tc_commit(mb2);
                }
                __syncwarp();
            }
            const bool has_next = c + 1 < nchunks;
            if (ok) ok = mbar_wait(mb2, c & 1);
            ok = all_ok(ok);
            tc_fence_after();
            tc_fence_before();
            bar_arrive(PP::EMPTY + stg, kEmptyCount);  // the stage's readers are done
            if (has_next) wait_gamma(c + 1);
            if (ok) state_pass(false, has_next ? sm.st[(c + 1) % PP::NS].gam : nullptr);
            tc_fence_before();
            bar_sync(bar_team, team_n);
        }
        if (OUT && hf == 1 && nchunks > 0) epilogue(nchunks - 1);
        cp_async_wait<0>();
        if (active && !ok && lane == 0 && p.err) atomicOr(p.err, 1);
    } else if (warp < 12) {
        // =========================================================== decay team
        const int d = tid - 256, sc = d >> 6, ip = 2 * (d & 63);
        const bf16 *beta = (const bf16 *)p.beta;
        const bf16 *vv = (const bf16 *)p.v;
        for (int cp = 0; cp < 6 && cp < nchunks; ++cp)  // the first chunks' v rows into L2
            if (d < 64 && kC * cp + (d >> 1) < len)
                prefetch_l2(vv + ((size_t)(t0 + kC * cp + (d >> 1)) * H + h) * kD + (d & 1) * 64);
        bool tok = true;
        auto load_beta = [&](int c) -> unsigned short {
            const int rows = min(kC, len - kC * c);
            return (c < nchunks && d < rows)
                       ? reinterpret_cast<const unsigned short *>(beta)[(size_t)(t0 + kC * c + d) * H + h]
                       : (unsigned short)0;
        };
        unsigned short bq = d < kC ? load_beta(0) : (unsigned short)0;
        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % PP::NS;
            unsigned char *R = sm.raw[c % PP::NR];
            Stage &St = sm.st[stg];
            const int rows = min(kC, len - kC * c);
            if (c >= PP::NS) bar_sync(PP::EMPTY + stg, kEmptyCount);  // the stage is free again
            {   // V tile of this chunk into the stage by cp.async, in the layout a
                // 128-byte-swizzled TMA box would have (MN-major A of MMA 1):
                // piece (row r, half hh, 16-byte chunk q) at hh*4096 + r*128 + (q ^ (r & 7))*16
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int x = d + 128 * i, r = x >> 4, hh = (x >> 3) & 1, q = x & 7;
                    const bool okr = r < rows;
                    cp_async16(St.v + hh * 4096 + r * 128 + ((q ^ (r & 7)) << 4),
                               vv + ((size_t)(t0 + kC * c + (okr ? r : 0)) * H + h) * kD + hh * 64 + q * 8, okr);
                }
                cp_async_commit();
                // the v rows of a later chunk into L2 (one 128-byte line per thread)
                const int cp = c + 6;
                if (d < 64 && cp < nchunks && kC * cp + (d >> 1) < len)
                    prefetch_l2(vv + ((size_t)(t0 + kC * cp + (d >> 1)) * H + h) * kD + (d & 1) * 64);
            }
            const unsigned short bq_next = d < kC ? load_beta(c + 1) : (unsigned short)0;
            if (d < kC) St.beta[d] = __bfloat162float(__ushort_as_bfloat16(bq));
            if (tok) tok = mbar_wait(smem_u32(&sm.mb_raw[c % PP::NR]), (c / PP::NR) & 1);
            if (rows < kC) {  // rows past the piece read as zero: decay 1, no write, no read
                const int n = (kC - rows) * 8;  // 16-byte pieces per tile half
                for (int x = d; x < 6 * n; x += 128) {
                    const int a = x / n, y = x % n;
                    const int hh = a & 1, tl = a >> 1;  // tl: 0 = k, 1 = g, 2 = q
                    if (!OUT && tl == 2) continue;
                    const int off = tl == 0 ? OFF_K : (tl == 1 ? OFF_G : OFF_Q);
                    *reinterpret_cast<uint4 *>(R + hh * kHalf + off + (rows + y / 8) * 128 + (y % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
            }
            __syncwarp();
            bar_sync(PP::DECAY, 128);
            // exp(g) and the inclusive prefix products over this tile's rows
            float2 e[16], E[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float2 gg = unpack_bf16(*reinterpret_cast<const uint32_t *>(R + rsw(OFF_G, 16 * sc + r, ip)));
                e[r] = make_float2(__expf(gg.x), __expf(gg.y));
            }
            {
                float2 acc = make_float2(1.f, 1.f);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    acc = f2mul(acc, e[r]);
                    E[r] = acc;
                }
            }
            const float2 gc = E[15];
            *reinterpret_cast<float2 *>(&sm.gexch[sc][ip]) = gc;
            bar_sync(PP::DECAY, 128);
            const float2 go = *reinterpret_cast<const float2 *>(&sm.gexch[sc ^ 1][ip]);
            const float2 g0 = sc ? go : gc, g1 = sc ? gc : go;
            if (sc == 0) {
                *reinterpret_cast<float2 *>(&St.gam[ip]) = f2mul(g0, g1);
                *reinterpret_cast<float2 *>(&sm.gam0[stg][ip]) = g0;
            }
            mbar_arrive(smem_u32(&sm.mb_gam[stg]));  // the state team may pre-scale with gamma
            const float2 inv = make_float2(__frcp_rn(gc.x), __frcp_rn(gc.y));
            const float2 kbs = sc ? make_float2(1.f, 1.f) : g1;  // Kbar scale of this tile
            const float2 qts = sc ? g0 : make_float2(1.f, 1.f);  // Q~ scale of this tile
            uint32_t kb0[8], kb1[8], qt0[8], qt1[8];  // Kbar / Q~ of channels ip, ip+1 (row pairs)
            {   // k: the tile column first (the in-place stores below would otherwise
                // keep every load behind the previous row's store), then suffix products
                uint32_t kr[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) kr[r] = *reinterpret_cast<const uint32_t *>(R + rsw(OFF_K, 16 * sc + r, ip));
                float2 F = make_float2(1.f, 1.f), kb_hi = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 15; r >= 0; --r) {
                    const int row = 16 * sc + r;
                    const float2 kv = unpack_bf16(kr[r]);
                    *reinterpret_cast<uint32_t *>(R + rsw(OFF_K, row, ip)) = pack_bf16(f2mul(kv, E[r]));
                    const float2 kF = f2mul(kv, F);
                    *reinterpret_cast<uint32_t *>(R + rsw(OFF_G, row, ip)) = pack_bf16(f2mul(kF, inv));
                    if (sc == 0) *reinterpret_cast<uint32_t *>(R + rsw(OFF_KB, r, ip)) = pack_bf16(kF);
                    const float2 kbv = f2mul(kF, kbs);
                    if (r & 1) {
                        kb_hi = kbv;
                    } else {
                        kb0[r >> 1] = pack_bf16(kbv.x, kb_hi.x);
                        kb1[r >> 1] = pack_bf16(kbv.y, kb_hi.y);
                    }
                    F = f2mul(F, e[r]);
                }
            }
            if (OUT) {  // q: needs only the prefix products
                uint32_t qr[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) qr[r] = *reinterpret_cast<const uint32_t *>(R + rsw(OFF_Q, 16 * sc + r, ip));
                const float2 sc2 = make_float2(p.scale, p.scale);
#pragma unroll
                for (int r = 0; r < 16; r += 2) {
                    const float2 qd0 = f2mul(f2mul(unpack_bf16(qr[r]), sc2), E[r]);
                    const float2 qd1 = f2mul(f2mul(unpack_bf16(qr[r + 1]), sc2), E[r + 1]);
                    *reinterpret_cast<uint32_t *>(R + rsw(OFF_Q, 16 * sc + r, ip)) = pack_bf16(qd0);
                    *reinterpret_cast<uint32_t *>(R + rsw(OFF_Q, 16 * sc + r + 1, ip)) = pack_bf16(qd1);
                    const float2 t0 = f2mul(qd0, qts), t1 = f2mul(qd1, qts);
                    qt0[r >> 1] = pack_bf16(t0.x, t1.x);
                    qt1[r >> 1] = pack_bf16(t0.y, t1.y);
                }
            }
            // Kbar^T rows ip, ip + 1 (K-major [128][32]): tokens 16 sc .. 16 sc + 15
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                *reinterpret_cast<uint4 *>(St.b2 + kmaj(ip, 16 * sc + 8 * hh, kC)) =
                    make_uint4(kb0[4 * hh], kb0[4 * hh + 1], kb0[4 * hh + 2], kb0[4 * hh + 3]);
                *reinterpret_cast<uint4 *>(St.b2 + kmaj(ip + 1, 16 * sc + 8 * hh, kC)) =
                    make_uint4(kb1[4 * hh], kb1[4 * hh + 1], kb1[4 * hh + 2], kb1[4 * hh + 3]);
            }
            // Q~ into columns 32 + 16 sc .. of [-W | Q~] (MN-major [K=128][N=64])
            if (OUT) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    *reinterpret_cast<uint4 *>(St.b1 + mnmaj(32 + 16 * sc + 8 * hh, ip, kD)) =
                        make_uint4(qt0[4 * hh], qt0[4 * hh + 1], qt0[4 * hh + 2], qt0[4 * hh + 3]);
                    *reinterpret_cast<uint4 *>(St.b1 + mnmaj(32 + 16 * sc + 8 * hh, ip + 1, kD)) =
                        make_uint4(qt1[4 * hh], qt1[4 * hh + 1], qt1[4 * hh + 2], qt1[4 * hh + 3]);
                }
            }
            cp_async_wait<0>();  // this thread's part of the V tile has landed
            fence_async_smem();  // tiles and stage are read by the tensor core next
            bar_sync(PP::DECAY, 128);
            // ---- AP: [Qd_0; Qd_1; Kd_0; Kd_1] x [Ki_0; Ki_1; Kb_0]^T (summary: [Kd_0; Kd_1; ...])
            // into AP buffer c % NS, issued as soon as the tiles are ready
            if (d < 32) {
                if (elect_one_sync()) {
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(R) + (OUT ? OFF_Q : OFF_K);
                    const uint32_t b0 = smem_u32(R) + OFF_G;
                    constexpr uint32_t ID_AP = idesc_bf16(64, 48, 0, 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                        tc_mma_ss(tbase + Cols<OUT>::AP + 64 * stg, sdesc_sw128(a0 + off, 16, 1024),
                                  sdesc_sw128(b0 + off, 16, 1024), ID_AP, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&sm.mb_ap[stg]));
                }
                __syncwarp();
            }
            bar_arrive(PP::DEC + c % PP::NR, kDecCount);
            bq = bq_next;
        }
        if (!tok && p.err) atomicOr(p.err, 2);
        // the stages of the last chunks come back before the CTA tears down
        for (int c = max(nchunks - PP::NS, 0); c < nchunks; ++c) bar_sync(PP::EMPTY + c % PP::NS, kEmptyCount);
    } else {
        // =========================================================== matrix team
        const int m = tid - 384, mw = m >> 5;
        const uint32_t lane_off = (uint32_t)(mw * 32) << 16;
        auto issue_raw = [&](int c) {
            unsigned char *R = sm.raw[c % PP::NR];
            const uint32_t mb = smem_u32(&sm.mb_raw[c % PP::NR]);
            const int tc = t0 + kC * c;
            mbar_arrive_expect_tx(mb, (OUT ? 3u : 2u) * 2u * 4096u);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t base = smem_u32(R) + hh * kHalf;
                tma_load_3d(base + OFF_K, &maps.k, 64 * hh, h, tc, mb);
                tma_load_3d(base + OFF_G, &maps.g, 64 * hh, h, tc, mb);
                if (OUT) tma_load_3d(base + OFF_Q, &maps.q, 64 * hh, h, tc, mb);
            }
        };
        if (m == 0)
            for (int c = 0; c < min(nchunks, PP::NR); ++c) issue_raw(c);
        // rows 32-63 of [T~ ; 0] (the O columns of MMA 1) and the block above
        // the diagonal of T~ (rows 0-15, columns 16-31) stay zero
        for (int x = m; x < PP::NS * 128; x += 128)
            reinterpret_cast<uint4 *>(sm.st[x >> 7].b0 + 2048)[x & 127] = make_uint4(0, 0, 0, 0);
        for (int x = m; x < PP::NS * 32; x += 128) {
            const int st = x >> 5, r = (x >> 1) & 15, hh = x & 1;
            *reinterpret_cast<uint4 *>(sm.st[st].b0 + kmaj(r, 16 + 8 * hh, kC)) = make_uint4(0, 0, 0, 0);
        }
        // the first chunks' tiles into L2
        auto prefetch = [&](int c) {
            if (c >= nchunks) return;
            const int tc = t0 + kC * c;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                tma_prefetch_3d(&maps.k, 64 * hh, h, tc);
                tma_prefetch_3d(&maps.g, 64 * hh, h, tc);
                if (OUT) tma_prefetch_3d(&maps.q, 64 * hh, h, tc);
            }
        };
        if (m == 0)
            for (int c = PP::NR; c < PP::NR + kPrefetch; ++c) prefetch(c);
        // A rows of the AP product: rows 32-63 in the output pass (after
        // Qd_0, Qd_1), rows 0-31 in the summary pass (no q)
        constexpr int kArow = OUT ? 2 : 0;
        constexpr uint32_t ID_W = idesc_bf16(128, 32, 1, 0);
        bool ok = true;

        for (int c = 0; c < nchunks; ++c) {
            const int stg = c % PP::NS;
            unsigned char *R = sm.raw[c % PP::NR];
            Stage &St = sm.st[stg];
            bar_sync(PP::DEC + c % PP::NR, kDecCount);  // Kd, Ki, Qd, Kb_0, beta, gamma of chunk c
            if (ok) ok = mbar_wait(smem_u32(&sm.mb_ap[stg]), (c / PP::NS) & 1);
            ok = all_ok(ok);
            tc_fence_after();
            const uint32_t col_ap = Cols<OUT>::AP + 64 * stg;
            if (ok) {
                // lanes 0-15 of quarter mw hold rows 16 mw .. 16 mw + 15 of D
                const uint32_t ta = tbase + lane_off + col_ap;
                const int rr = lane;  // row within the 16-row block (lanes >= 16 idle)
                if (mw == kArow) {  // rows of Kd_0: A00 (strictly lower)
                    uint32_t a[16];
                    tmem_ld16(ta, a);
                    tc_wait_ld();
                    if (rr < 16) {
                        const float b = St.beta[rr];
#pragma unroll
                        for (int s = 0; s < kC; ++s)
                            sm.AT[s * kC + rr] = (s < rr) ? b * __uint_as_float(a[s & 15]) : 0.f;
                    }
                } else if (mw == kArow + 1) {  // rows of Kd_1: A10 (cols 32-47), A11 (cols 16-31)
                    uint32_t a[32];
                    tmem_ld32(ta + 16, a);
                    tc_wait_ld();
                    if (rr < 16) {
                        const int r = 16 + rr;
                        const float b = St.beta[r];
#pragma unroll
                        for (int s = 0; s < kC; ++s) {
                            const float x = s < 16 ? __uint_as_float(a[16 + s])
                                                   : (s - 16 < rr ? __uint_as_float(a[s - 16]) : 0.f);
                            sm.AT[s * kC + r] = b * x;
                        }
                    }
                } else if (OUT && mw == 0) {  // rows of Qd_0: P00 (lower, diagonal in)
                    uint32_t a[16];
                    tmem_ld16(ta, a);
                    tc_wait_ld();
                    if (rr < 16) {
                        uint32_t pk[16];
#pragma unroll
                        for (int s2 = 0; s2 < 16; ++s2) {
                            const int s = 2 * s2;
                            const float x0 = (s < 16 && s <= rr) ? __uint_as_float(a[s & 15]) : 0.f;
                            const float x1 = (s + 1 < 16 && s + 1 <= rr) ? __uint_as_float(a[(s + 1) & 15]) : 0.f;
                            pk[s2] = pack_bf16(x0, x1);
                        }
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4 *>(St.b3 + kmaj(rr, 8 * q4, kC)) =
                                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                    }
                } else if (OUT && mw == 1) {  // rows of Qd_1: P10 (cols 32-47), P11 (cols 16-31)
                    uint32_t a[32];
                    tmem_ld32(ta + 16, a);
                    tc_wait_ld();
                    if (rr < 16) {
                        uint32_t pk[16];
#pragma unroll
                        for (int s2 = 0; s2 < 16; ++s2) {
                            const int s = 2 * s2;
                            auto pv = [&](int ss) {
                                return ss < 16 ? __uint_as_float(a[16 + ss])
                                               : (ss - 16 <= rr ? __uint_as_float(a[ss - 16]) : 0.f);
                            };
                            pk[s2] = pack_bf16(pv(s), pv(s + 1));
                        }
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4 *>(St.b3 + kmaj(16 + rr, 8 * q4, kC)) =
                                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            bar_sync(PP::MAT, 128);
            // ---- T = (I + N)^-1, N = Diag(beta) A, by blocks: the two 16 x 16
            // diagonal blocks by forward substitution on one warp (lane l:
            // block l / 16, column l % 16; once row r is final it is pushed into
            // every later row), then T10 = -T11 (N10 T00) by all 128 threads,
            // fp32 throughout.  T~ = T Diag(beta) into [T~ ; 0] as bf16.
            if (mw == 0 && ok) {
                const int blk = lane >> 4, jj = lane & 15, o = 16 * blk;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == jj) ? 1.f : 0.f;
#pragma unroll
                for (int r = 0; r < 15; ++r) {
                    float at[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(&sm.AT[(o + r) * kC + o + 4 * q4]);
                        at[4 * q4 + 0] = a4.x; at[4 * q4 + 1] = a4.y;
                        at[4 * q4 + 2] = a4.z; at[4 * q4 + 3] = a4.w;
                    }
#pragma unroll
                    for (int r2 = r + 1; r2 < 16; ++r2) x[r2] = fmaf(-at[r2], x[r], x[r2]);
                }
                const float bj = St.beta[o + jj];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    sm.Td[blk][r * 16 + jj] = x[r];
                    *reinterpret_cast<bf16 *>(St.b0 + kmaj(o + r, o + jj, kC)) = __float2bfloat16_rn(x[r] * bj);
                }
            }
            bar_sync(PP::MAT, 128);
            const int zi = m >> 3, zj = 2 * (m & 7);  // this thread's two entries of the 16 x 16 products
            if (ok) {  // Z = N10 T00, N10[i][s] = AT[s][16 + i]
                float2 z = make_float2(0.f, 0.f);
#pragma unroll
                for (int s2 = 0; s2 < 16; ++s2) {
                    const float n = sm.AT[s2 * kC + 16 + zi];
                    const float2 t = *reinterpret_cast<const float2 *>(&sm.Td[0][s2 * 16 + zj]);
                    z.x = fmaf(n, t.x, z.x);
                    z.y = fmaf(n, t.y, z.y);
                }
                *reinterpret_cast<float2 *>(&sm.Zx[zi * 16 + zj]) = z;
            }
            bar_sync(PP::MAT, 128);
            if (ok) {  // T10 = -T11 Z;  T~10 = T10 Diag(beta_0)
                float2 t10 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k2 = 0; k2 < 16; ++k2) {
                    const float t11 = sm.Td[1][zi * 16 + k2];
                    const float2 z = *reinterpret_cast<const float2 *>(&sm.Zx[k2 * 16 + zj]);
                    t10.x = fmaf(t11, z.x, t10.x);
                    t10.y = fmaf(t11, z.y, t10.y);
                }
                *reinterpret_cast<uint32_t *>(St.b0 + kmaj(16 + zi, zj, kC)) =
                    pack_bf16(-t10.x * St.beta[zj], -t10.y * St.beta[zj + 1]);
            }
            fence_async_smem();
            tc_fence_before();
            bar_sync(PP::MAT, 128);
            // ---- W^T = Kd_0^T T~[:, 0:16]^T + Diag(gamma_0) Kd_1^T T~[:, 16:32]^T,
            // into this chunk's AP buffer (its Gram blocks have been read out)
            if (mw == 0 && ok) {
                if (elect_one_sync()) {
                    tc_fence_after();
                    const uint32_t kt = smem_u32(R) + OFF_K;
                    const uint32_t bt = smem_u32(St.b0);
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt)  // tile tt: rows 16 tt .. of the k tile, columns 16 tt .. of T~
                        tc_mma_ss(tbase + col_ap + 32 * tt, sdesc_sw128(kt + 2048 * tt, kHalf, 1024),
                                  sdesc(bt + 256 * tt, 128, 512), ID_W, 0u);
                    tc_commit(smem_u32(&sm.mb_w));
                }
                __syncwarp();
            }
            if (ok) ok = mbar_wait(smem_u32(&sm.mb_w), c & 1);
            ok = all_ok(ok);
            tc_fence_after();
            if (ok) {  // thread m = key channel i: -W[t][i] into row i of [-W | Q~]
                uint32_t xa[32], ya[32];
                const uint32_t tw = tbase + lane_off + col_ap;
                tmem_ld32(tw, xa);
                tmem_ld32(tw + 32, ya);
                tc_wait_ld();
                const float g0 = sm.gam0[stg][m];
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const int t = 8 * q8 + 2 * e2;
                        w4[e2] = pack_bf16(-fmaf(g0, __uint_as_float(ya[t]), __uint_as_float(xa[t])),
                                           -fmaf(g0, __uint_as_float(ya[t + 1]), __uint_as_float(xa[t + 1])));
                    }
                    *reinterpret_cast<uint4 *>(St.b1 + mnmaj(8 * q8, m, kD)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            bar_sync(PP::MAT, 128);  // every read of the raw tiles and of gam0 is done
            if (m == 0) {
                if (c + PP::NR < nchunks) issue_raw(c + PP::NR);
                prefetch(c + PP::NR + kPrefetch);
            }
            bar_arrive(PP::FULL + stg, kFullCount);
        }
        if (!ok && m == 0 && p.err) atomicOr(p.err, 2);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(512) : "memory");
}

// Summary pass: one CTA per (piece, head) that has a successor (or every
// piece when all maps are asked for); the head is the fastest grid index so
// co-resident CTAs cover all heads of a few pieces.
__global__ void __launch_bounds__(kThreads, 1) summary_kernel(PrefillParams p, const __grid_constant__ Maps maps) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    const bool want_s = p.summarize_all || j < np - 1;
    const bool want_m = p.summarize_all || (j > 0 && j < np - 1);
    if (!want_s && !want_m) return;
    const size_t ph = (size_t)pi * p.H + h;
    const float *init = (j == 0 && p.initial_state) ? p.initial_state + ((size_t)n * p.H + h) * kD * kD : nullptr;
    run_piece<false>(p, maps, pc.y, pc.z, h, init, want_s ? p.Szero + ph * kD * kD : nullptr,
                     want_m ? p.M + ph * kD * kD : nullptr, smem);
}

__global__ void __launch_bounds__(kThreads, 1) output_kernel(PrefillParams p, const __grid_constant__ Maps maps) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int h = blockIdx.x % p.H, pi = blockIdx.x / p.H;
    const int4 pc = p.pieces[pi];
    if (pc.x < 0) return;
    const int n = pc.x, j = pc.w;
    const int np = p.seq_first[n + 1] - p.seq_first[n];
    const size_t nh = (size_t)n * p.H + h;
    const float *init = (np == 1) ? (p.initial_state ? p.initial_state + nh * kD * kD : nullptr)
                                  : p.Sin + ((size_t)pi * p.H + h) * kD * kD;
    float *fin = (j == np - 1 && p.final_state) ? p.final_state + nh * kD * kD : nullptr;
    run_piece<true>(p, maps, pc.y, pc.z, h, init, fin, nullptr, smem);
}

}  // namespace c32

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// [T][H][128] bf16 as a 3-D tensor (channel, head, token), boxes of 32 tokens:
// 64 channels with the 128-byte swizzle, or all 128 without swizzle.
bool encode(CUtensorMap *m, const void *base, int T, int H, bool swizzled) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {256, (cuuint64_t)H * 256};
    const cuuint32_t box[3] = {swizzled ? 64u : 128u, 1, 32};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

// bf16, dk = dv = 128, no extended features, pieces a multiple of 32 tokens.
cudaError_t launch_prefill_c32(const PrefillParams &p, bool summaries, cudaStream_t st) {
    c32::Maps maps;
    memset(&maps, 0, sizeof(maps));
    const int T = p.total_tokens, H = p.H;
    if (T > 0) {
        bool ok = encode(&maps.k, p.k, T, H, true) && encode(&maps.g, p.g, T, H, true);
        if (!summaries) ok = ok && encode(&maps.q, p.q, T, H, true);
        if (!ok) return cudaErrorInvalidValue;
    }
    const dim3 grid((unsigned)(p.P_max * p.H));
    cudaError_t e;
    if (summaries) {
        const size_t sm = c32::kSmemBytes<false>;
        e = cudaFuncSetAttribute(c32::summary_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        c32::summary_kernel<<<grid, c32::kThreads, sm, st>>>(p, maps);
    } else {
        const size_t sm = c32::kSmemBytes<true>;
        e = cudaFuncSetAttribute(c32::output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        c32::output_kernel<<<grid, c32::kThreads, sm, st>>>(p, maps);
    }
    return cudaGetLastError();
}

}  // namespace kda
