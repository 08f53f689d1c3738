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
// With sub-pieces (the 16-token tcgen05 kernels, when the plan asks for
// them) the summary runs over pieces cut into `sub` equal parts, which fills
// the summary pass's waves better, and a fold composes each piece's sub-piece
// maps into the piece's (M, S_zero) before the scan:
//   plan, plan of the sub-pieces, summary (sub-pieces), fold, scan, output.
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
// and, with sub-pieces (P_sub_max > 0), the same plan sections and the two
// maps once more for the sub-pieces.
struct WorkspaceLayout {
    size_t off_header, off_seq_first, off_pieces, off_M, off_Szero, off_Sin;
    size_t off_header_sub, off_seq_first_sub, off_pieces_sub, off_M_sub, off_Szero_sub, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(long P_max, int num_seqs, int H, int dk, int dv, long P_sub_max = 0) {
    WorkspaceLayout L;
    size_t o = 0;
    L.off_header = o;    o = align256(o + 64 * sizeof(int32_t));
    L.off_seq_first = o; o = align256(o + (size_t)(num_seqs + 1) * sizeof(int32_t));
    L.off_pieces = o;    o = align256(o + (size_t)P_max * 4 * sizeof(int32_t));
    L.off_M = o;         o = align256(o + (size_t)P_max * H * dk * dk * sizeof(float));
    L.off_Szero = o;     o = align256(o + (size_t)P_max * H * dk * dv * sizeof(float));
    L.off_Sin = o;       o = align256(o + (size_t)P_max * H * dk * dv * sizeof(float));
    L.off_header_sub = L.off_seq_first_sub = L.off_pieces_sub = L.off_M_sub = L.off_Szero_sub = o;
    if (P_sub_max > 0) {
        L.off_header_sub = o;    o = align256(o + 64 * sizeof(int32_t));
        L.off_seq_first_sub = o; o = align256(o + (size_t)(num_seqs + 1) * sizeof(int32_t));
        L.off_pieces_sub = o;    o = align256(o + (size_t)P_sub_max * 4 * sizeof(int32_t));
        L.off_M_sub = o;         o = align256(o + (size_t)P_sub_max * H * dk * dk * sizeof(float));
        L.off_Szero_sub = o;     o = align256(o + (size_t)P_sub_max * H * dk * dv * sizeof(float));
    }
    L.total = o;
    return L;
}

// ---------------------------------------------------------------- the plan
// Piece length (tokens, a multiple of the kernels' chunk).  Each (piece, head)
// is one CTA of the output pass, so its time is counted in whole waves of
// `slots_out` CTAs.  A sequence of p > 1 pieces costs an output pass over all
// p pieces, a summary pass over pieces 0..p-2 (one CTA per (piece, head)
// computes both the zero-start state and the transition; waves of
// `slots_sum`) and p - 1 steps of the prefix scan.  With sub-pieces, each
// summarised piece is cut into `sub` equal parts summarised by separate CTAs
// (shorter CTAs fill the summary's waves better) and `sub` - 1 fold steps
// compose their maps.  With equal-length sequences (the lengths are not known
// on the host in general) the model is
//   cost(L, sub) = waves(output) * chunks(L)
//                  + sum_ratio * waves(summary units) * chunks(L) / sub
//                  + scan_cost * (pieces - 1) + fold_cost * (sub - 1)
// in units of one chunk step of the output pass.  When the host copy of the
// offsets is given, the real lengths are used, and only plans whose tables fit
// the workspace sized for the length-blind choice are considered.
struct PlanModel {
    int chunk;          // tokens per chunk step (16 or 32); pieces are multiples of it
    long slots_out;     // output-pass CTAs resident at once
    long slots_sum;     // summary-pass CTAs resident at once
    double sum_ratio;   // summary chunk step / output chunk step
    double scan_cost;   // one scan step, in output chunk steps
    int sub_max;        // most sub-pieces a summarised piece may be cut into (1 = none)
    double fold_cost;   // one fold step, in output chunk steps
};
// The 16-token kernels: output pass two CTAs per SM, the paired summary one;
// 0.67 is the measured ratio of their per-chunk periods at full occupancy
// (about 2.96 K and 4.44 K SM cycles), a scan step about two output chunk
// steps, a fold step about thirteen (measured: 87 us for the three steps of
// 256 piece-head chains, one output chunk step being about 2.2 us).
// Sub-pieces are for the tcgen05 kernels only (the caller clears sub_max for
// the others).
inline PlanModel plan_model_chunk16(int sms) { return PlanModel{16, 2L * sms, (long)sms, 0.67, 2.0, 4, 13.0}; }
// The 32-token kernels (bf16, dk = dv = 128): both passes one CTA per SM.
inline PlanModel plan_model_chunk32(int sms) { return PlanModel{32, (long)sms, (long)sms, 1.0, 6.0, 1, 0.0}; }

struct PlanChoice {
    long piece_len;
    int sub;  // sub-pieces per summarised piece (1 = none)
};

inline long max_pieces_of(long total_tokens, int num_seqs, long piece_len) {
    return (long)num_seqs + (total_tokens + piece_len - 1) / piece_len;
}

inline double plan_cost(long L, int sub, int num_seqs, int H, const PlanModel &pm, const int32_t *cu_host,
                        long total_tokens) {
    long out = 0, sum = 0, max_chunks = 0, max_pieces = 1;
    for (int n = 0; n < (cu_host ? num_seqs : 1); ++n) {
        const long len = cu_host ? (long)cu_host[n + 1] - cu_host[n]
                                 : (total_tokens + num_seqs - 1) / num_seqs;
        const long pcs = len <= 0 ? 1 : (len + L - 1) / L;
        const long mult = cu_host ? 1 : num_seqs;
        out += mult * pcs;
        sum += mult * (pcs - 1) * sub;
        const long ch = (std::min(len, L) + pm.chunk - 1) / pm.chunk;
        if (ch > max_chunks) max_chunks = ch;
        if (pcs > max_pieces) max_pieces = pcs;
    }
    const long w_out = (out * H + pm.slots_out - 1) / pm.slots_out;
    const long sum_slots = std::max(pm.slots_sum, 1L);
    const long w_sum = (sum * H + sum_slots - 1) / sum_slots;
    return (double)w_out * max_chunks + pm.sum_ratio * (double)w_sum * (double)((max_chunks + sub - 1) / sub) +
           pm.scan_cost * (double)(max_pieces - 1) +
           (sub > 1 && max_pieces > 1 ? pm.fold_cost * (double)(sub - 1) : 0.0);
}

inline long env_positive(const char *name) {
    const char *s = getenv(name);
    if (!s || !*s) return 0;
    char *end = nullptr;
    const long v = strtol(s, &end, 10);
    return (end && *end == 0 && v > 0) ? v : 0;
}

// KDA_PIECE_LEN forces the piece length (rounded up to whole chunks, and to
// whole sub-pieces); KDA_SUB_PIECES forces the number of sub-pieces (at most
// sub_max).
inline PlanChoice plan_choose(long total_tokens, int num_seqs, int H, const PlanModel &pm_in,
                              const int32_t *cu_host) {
    const long C = pm_in.chunk;
    const int sub_max = std::max(pm_in.sub_max, 1);
    const long forced_sub = std::min<long>(env_positive("KDA_SUB_PIECES"), sub_max);
    const long forced = env_positive("KDA_PIECE_LEN");
    if (forced > 0) {
        const long m = forced_sub > 0 ? forced_sub : 1;
        return PlanChoice{((forced + C * m - 1) / (C * m)) * C * m, (int)m};
    }
    PlanModel pm = pm_in;
    if (env_positive("KDA_SLOTS")) pm.slots_out = env_positive("KDA_SLOTS");
    if (num_seqs <= 0 || total_tokens <= 0) return PlanChoice{256, 1};
    // floors: the chosen tables must fit the workspace of the length-blind plan
    auto search = [&](const int32_t *cu, long Lref, const PlanChoice *floor) {
        PlanChoice best{0, 1};
        double best_cost = 0;
        for (int m = 1; m <= sub_max; m *= 2) {
            if (forced_sub > 0 && m != forced_sub) continue;
            if (floor && m > 1 && floor->sub == 1) continue;  // no sub-piece tables in the workspace
            for (int pcs = 1; pcs <= 128; ++pcs) {
                long L = ((Lref + pcs - 1) / pcs + C * m - 1) / (C * m) * (C * m);
                L = std::max<long>(L, ((256 + C * m - 1) / (C * m)) * C * m);
                if (floor) {
                    if (L < floor->piece_len) break;
                    if (m > 1 && L / m < floor->piece_len / floor->sub) break;
                }
                const double c = plan_cost(L, m, num_seqs, H, pm, cu, total_tokens);
                if (best.piece_len == 0 || c < best_cost) {
                    best = PlanChoice{L, m};
                    best_cost = c;
                }
                if (L <= ((256 + C * m - 1) / (C * m)) * C * m) break;
            }
        }
        if (best.piece_len == 0) best = floor ? *floor : PlanChoice{std::max<long>(((Lref + C - 1) / C) * C, 256), 1};
        return best;
    };
    const long Lavg = (total_tokens + num_seqs - 1) / num_seqs;
    PlanChoice blind = search(nullptr, Lavg, nullptr);
    blind.piece_len = std::min<long>(blind.piece_len, 1L << 30);
    // the exact model walks every sequence per candidate: only for modest N
    if (!cu_host || num_seqs > 8192) return blind;
    long Lmax = 0;
    for (int n = 0; n < num_seqs; ++n) Lmax = std::max<long>(Lmax, (long)cu_host[n + 1] - cu_host[n]);
    PlanChoice c = search(cu_host, std::max(Lmax, blind.piece_len), &blind);
    c.piece_len = std::min<long>(c.piece_len, 1L << 30);
    return c;
}

// The plan without sub-pieces (callers whose kernels do not take them).
inline int plan_piece_len(long total_tokens, int num_seqs, int H, const PlanModel &pm_in,
                          const int32_t *cu_host) {
    PlanModel pm = pm_in;
    pm.sub_max = 1;
    return (int)plan_choose(total_tokens, num_seqs, H, pm, cu_host).piece_len;
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
    // summary launches over sub-pieces: the pieces table holds sub-pieces,
    // `sub` of them per piece of the output pass (0 or 1 = plain pieces)
    int sub;
};

// The fold of sub-piece maps into piece maps (plans with sub-pieces): the
// output pass's piece table and the sub-piece table in, the sub-piece maps
// in, the piece maps (what the scan reads) out.
struct SubFoldParams {
    const int4 *pieces;
    const int32_t *seq_first, *seq_first_sub;
    const float *M_sub, *Z_sub;
    float *M, *Z;
    int H, P_max, P_sub_max, sub;
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
// The call runs the 16-token tcgen05 kernels (the only ones that summarise
// sub-pieces).
inline bool tc5_path(bool bf16, int dk, int dv, int flags, int snap_tokens) {
    const int f = prefill_impl_forced();
    return bf16 && dk == 128 && dv == 128 && f != 3 && f != 4 && !chunk32_eligible(bf16, dk, dv, flags, snap_tokens);
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
