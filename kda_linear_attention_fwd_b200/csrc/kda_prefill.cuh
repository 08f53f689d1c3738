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

namespace kda {

constexpr int kChunk = 16;

// Workspace layout (all offsets 256-byte aligned), for P_max pieces:
//   int32 plan header [64]           : [0] = number of pieces P
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
    int num_seqs, H, P_max;
    float scale;
    int qk_l2norm;
};

}  // namespace kda
