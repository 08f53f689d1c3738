// KDA prefill: shared definitions of the piece plan and the launch parameters.
//
// Two-level chunking (prism.simon-ai.net, "从架构创新出发：K3的MoE与混合注意力设计",
// section "Linear Attention 的分层 Chunking 策略"; affta.cn K3 explainer,
// section "KDA 上下文并行，让上下文的交接变薄"):
//
//   * inner level: 16-token chunks, inside which the work is whole-block
//     matrix products and between which the state is carried;
//   * outer level: each sequence is cut into pieces of `piece_len` tokens
//     (a multiple of 16, counted from the sequence start).  A piece's effect
//     on the state is affine, S_out = M S_in + S_zero, where M (dk x dk) says
//     how the piece transforms an incoming state and S_zero is the state it
//     produces from zero.  Pieces summarise themselves in parallel, a prefix
//     scan over the pieces of a sequence turns the summaries into each
//     piece's incoming state, and every piece then runs again from its
//     incoming state to produce its outputs.
//
// Launch sequence of kda_chunk_fwd (one stream):
//   plan     -> piece table from cu_seqlens
//   summary  -> (M, S_zero) of every piece that has a successor
//   scan     -> incoming state of every piece (sequences with >1 piece)
//   output   -> every piece from its incoming state: y, and the final state
// When no sequence can have more than one piece, only plan and output run.
#pragma once

#include <stdint.h>
#include <stdlib.h>

#include <algorithm>

namespace kda {

constexpr int kChunk = 16;

// Workspace layout (all offsets 256-byte aligned), for P_max pieces:
//   int32 plan header [64]           : [0] = number of pieces P, [1] = offsets
//                                      inconsistent, [2] = device wait timed out
//   int32 seq_first   [num_seqs + 1] : first piece of each sequence
//   int4  pieces      [P_max]        : {seq, token start, length, index in seq}
//   fp32  M           [P_max][H][dk][dk]   transition of each piece
//   fp32  Szero       [P_max][H][dk][dv]   state each piece makes from zero
//   fp32  Sin         [P_max][H][dk][dv]   incoming state of each piece
struct WorkspaceLayout {
    size_t off_header, off_seq_first, off_pieces, off_M, off_Szero, off_Sin, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(long P_max, int num_seqs, int H, int dk, int dv) {
    WorkspaceLayout L;
    size_t o = 0;
    L.off_header = o;    o = align256(o + 64 * sizeof(int32_t));
    L.off_seq_first = o; o = align256(o + (size_t)(num_seqs + 1) * sizeof(int32_t));
    L.off_pieces = o;    o = align256(o + (size_t)P_max * 4 * sizeof(int32_t));
    L.off_M = o;         o = align256(o + (size_t)P_max * H * dk * dk * sizeof(float));
    L.off_Szero = o;     o = align256(o + (size_t)P_max * H * dk * dv * sizeof(float));
    L.off_Sin = o;       o = align256(o + (size_t)P_max * H * dk * dv * sizeof(float));
    L.total = o;
    return L;
}

// ---------------------------------------------------------------- the plan
// Piece length (tokens, a multiple of the kernels' chunk).  Each (piece, head)
// is one CTA of the output pass, so its time is counted in whole waves of
// `slots_out` CTAs.  A sequence of p > 1 pieces costs an output pass over all
// p pieces, a summary pass over pieces 0..p-2 (one CTA per (piece, head)
// computes both the zero-start state and the transition; waves of
// `slots_sum`) and p - 1 steps of the prefix scan.  With equal-length
// sequences (the lengths are not known on the host in general) the model is
//   cost(L) = waves(output) * chunks(L) + sum_ratio * waves(summary) * chunks(L)
//             + scan_cost * (pieces - 1)
// in units of one chunk step of the output pass.  When the host copy of the
// offsets is given, the real lengths are used, and only piece lengths at
// least as long as the length-blind choice are considered, so that the
// workspace sized without the lengths still fits.
struct PlanModel {
    int chunk;          // tokens per chunk step (16 or 32); pieces are multiples of it
    long slots_out;     // output-pass CTAs resident at once
    long slots_sum;     // summary-pass CTAs resident at once
    double sum_ratio;   // summary chunk step / output chunk step
    double scan_cost;   // one scan step, in output chunk steps
};
// The 16-token kernels: output pass two CTAs per SM, the paired summary one;
// 0.67 is the measured ratio of their per-chunk periods at full occupancy
// (about 2.96 K and 4.44 K SM cycles), a scan step about two output chunk
// steps.
inline PlanModel plan_model_chunk16(int sms) { return PlanModel{16, 2L * sms, (long)sms, 0.67, 2.0}; }
// The 32-token kernels (bf16, dk = dv = 128): both passes one CTA per SM.
inline PlanModel plan_model_chunk32(int sms) { return PlanModel{32, (long)sms, (long)sms, 1.0, 6.0}; }

inline double plan_cost(long L, int num_seqs, int H, const PlanModel &pm, const int32_t *cu_host,
                        long total_tokens) {
    long out = 0, sum = 0, max_chunks = 0, max_pieces = 1;
    for (int n = 0; n < (cu_host ? num_seqs : 1); ++n) {
        const long len = cu_host ? (long)cu_host[n + 1] - cu_host[n]
                                 : (total_tokens + num_seqs - 1) / num_seqs;
        const long pcs = len <= 0 ? 1 : (len + L - 1) / L;
        const long mult = cu_host ? 1 : num_seqs;
        out += mult * pcs;
        sum += mult * (pcs - 1);
        const long ch = (std::min(len, L) + pm.chunk - 1) / pm.chunk;
        if (ch > max_chunks) max_chunks = ch;
        if (pcs > max_pieces) max_pieces = pcs;
    }
    const long w_out = (out * H + pm.slots_out - 1) / pm.slots_out;
    const long sum_slots = std::max(pm.slots_sum, 1L);
    const long w_sum = (sum * H + sum_slots - 1) / sum_slots;
    return (double)w_out * max_chunks + pm.sum_ratio * (double)w_sum * max_chunks +
           pm.scan_cost * (double)(max_pieces - 1);
}

inline long env_positive(const char *name) {
    const char *s = getenv(name);
    if (!s || !*s) return 0;
    char *end = nullptr;
    const long v = strtol(s, &end, 10);
    return (end && *end == 0 && v > 0) ? v : 0;
}

inline int plan_piece_len(long total_tokens, int num_seqs, int H, const PlanModel &pm_in,
                          const int32_t *cu_host) {
    const long C = pm_in.chunk;
    const long forced = env_positive("KDA_PIECE_LEN");
    if (forced > 0) return (int)(((forced + C - 1) / C) * C);
    PlanModel pm = pm_in;
    if (env_positive("KDA_SLOTS")) pm.slots_out = env_positive("KDA_SLOTS");
    if (num_seqs <= 0 || total_tokens <= 0) return 256;
    auto search = [&](const int32_t *cu, long Lref, long L_floor) {
        long best_L = std::max<long>(((Lref + C - 1) / C) * C, 256);
        best_L = std::max(best_L, L_floor);
        double best = plan_cost(best_L, num_seqs, H, pm, cu, total_tokens);
        for (int pcs = 2; pcs <= 128; ++pcs) {
            long L = ((Lref + pcs - 1) / pcs + C - 1) / C * C;
            if (L < 256 || L < L_floor) break;
            const double c = plan_cost(L, num_seqs, H, pm, cu, total_tokens);
            if (c < best) { best = c; best_L = L; }
        }
        return best_L;
    };
    const long Lavg = (total_tokens + num_seqs - 1) / num_seqs;
    const long L_blind = search(nullptr, Lavg, 0);
    // the exact model walks every sequence per candidate: only for modest N
    if (!cu_host || num_seqs > 8192) return (int)std::min<long>(L_blind, 1L << 30);
    long Lmax = 0;
    for (int n = 0; n < num_seqs; ++n) Lmax = std::max<long>(Lmax, (long)cu_host[n + 1] - cu_host[n]);
    return (int)std::min<long>(search(cu_host, std::max(Lmax, L_blind), L_blind), 1L << 30);
}

struct PrefillParams {
    const void *q, *k, *v, *g, *beta, *gate;
    void *out;
    const int32_t *cu_seqlens;
    const int32_t *header;
    const int32_t *seq_first;
    const int4 *pieces;
    float *M, *Szero, *Sin;
    const float *initial_state;
    float *final_state;
    int32_t *err;  // header[2]: set to nonzero when a bounded device wait gave up
    int num_seqs, H, P_max;
    int total_tokens;
    float scale;
    int flags;                    // FLAG_* bits (kda_common.cuh)
    // state snapshots after every snap_tokens tokens of a sequence (0 = none):
    // snapshot m (m = 1, 2, ... while m * snap_tokens < length) of sequence n
    // and head h at snapshots[((snap_offsets[n] + m - 1) * H + h) * dk * dv]
    int snap_tokens;
    float *snapshots;
    const int32_t *snap_offsets;
    // summary pass over every piece (both parts), for the per-sequence affine
    // map of kda_chunk_fwd_summary; 0 = the prefill's own summary pass
    int summarize_all;
    // piece length of the plan (tokens): the 32-token kernels need a multiple of 32
    int piece_len;
};

// The 32-token kernels (bf16, dk = dv = 128, none of the extended features)
// run when KDA_PREFILL_IMPL=c32 asks for them; by default every call runs in
// 16-token chunks, which measured faster on B200 (two CTAs per SM against
// one).  KDA_PREFILL_IMPL (c32 | tc5 | mma | simt) forces a path where it
// applies.
inline int prefill_impl_forced() {
    const char *e = getenv("KDA_PREFILL_IMPL");
    if (!e || !*e) return 0;
    if (e[0] == 'c') return 1;
    if (e[0] == 't') return 2;
    if (e[0] == 'm') return 3;
    if (e[0] == 's') return 4;
    return 0;
}
inline bool chunk32_eligible(bool bf16, int dk, int dv, int flags, int snap_tokens) {
    const int f = prefill_impl_forced();
    return bf16 && dk == 128 && dv == 128 && flags == 0 && snap_tokens == 0 && f == 1;
}

// Where the output pass of one (piece, head) writes state snapshots.
struct Snap {
    float *base = nullptr;  // first snapshot of this (sequence, head); null = none
    size_t stride = 0;      // floats between consecutive snapshots of it
    int pos0 = 0;           // position of the piece's first token in its sequence
    int len = 0;            // sequence length
    int every = 0;          // snapshot interval in tokens (a multiple of 16)
    // The state after position pos_end - 1 goes here, or nowhere (null).
    __device__ __forceinline__ float *at(int pos_end) const {
        if (!base || pos_end % every != 0 || pos_end >= len) return nullptr;
        return base + (size_t)(pos_end / every - 1) * stride;
    }
};
__device__ __forceinline__ Snap make_snap(const PrefillParams &p, int n, int h, int t0, size_t dkdv) {
    Snap sn;
    if (p.snap_tokens > 0 && p.snapshots && p.snap_offsets) {
        const int a = p.cu_seqlens[n], b = p.cu_seqlens[n + 1];
        sn.base = p.snapshots + ((size_t)p.snap_offsets[n] * p.H + h) * dkdv;
        sn.stride = (size_t)p.H * dkdv;
        sn.pos0 = t0 - a;
        sn.len = b - a;
        sn.every = p.snap_tokens;
    }
    return sn;
}

}  // namespace kda
