// C-ABI entry points of libkda_b200.so (declared in include/kda.h): argument
// validation, the piece plan, and the launch sequence.  No allocation, no
// host synchronisation, no exceptions across the boundary.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "../../include/kda.h"
#include "kda_args.h"
#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {
cudaError_t launch_decode(bool bf16, int dk, int dv, const void *q, const void *k, const void *v,
                          const void *g, const void *beta, const void *gate, void *out,
                          float *state, long nh, float scale, int l2, cudaStream_t st);
cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st);
cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st);
cudaError_t launch_subfold_tc(const SubFoldParams &p, int32_t *err, cudaStream_t st);
cudaError_t launch_prefill_chunks(const PrefillParams &p, bool bf16, int dk, int dv,
                                  bool summaries, cudaStream_t st);

#ifdef KDA_CHECK_G
// Checked builds: the log-decay precondition ln(0.0067) <= g <= 0 (with the
// clamp flag only g <= 0, the kernels raise smaller values to the floor);
// NaN fails either test.  A violation sets bit 4 of the workspace error word.
template <typename T>
__global__ void __launch_bounds__(256) check_g_kernel(const T *g, long n, int clamp, int32_t *err) {
    bool bad = false;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const float x = ld(g + i);
        bad |= !(x <= 0.f && (clamp || x >= kLogDecayFloor));
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, 4);
}

cudaError_t launch_check_g(const void *g, bool bf16, long n, int clamp, int32_t *err,
                           cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const unsigned blocks = (unsigned)std::min<long>((n + 255) / 256, 1184);
    if (bf16)
        check_g_kernel<<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)g, n, clamp, err);
    else
        check_g_kernel<<<blocks, 256, 0, st>>>((const float *)g, n, clamp, err);
    return cudaGetLastError();
}
#endif
}  // namespace kda

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128; }

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev < 0 || dev >= 64) dev = 0;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

enum class Path { chunk16, tc5, chunk32 };  // kernel families with their own plans

// The plan of a call on one kernel family: sub-pieces only for the 16-token
// tcgen05 kernels.
kda::PlanChoice choose_plan(long total_tokens, int num_seqs, int H, Path path,
                            const int32_t *cu_host = nullptr) {
    kda::PlanModel pm = path == Path::chunk32 ? kda::plan_model_chunk32(sm_count())
                                              : kda::plan_model_chunk16(sm_count());
    if (path != Path::tc5) pm.sub_max = 1;
    kda::PlanChoice c = kda::plan_choose(total_tokens, num_seqs, H, pm, cu_host);
    if (c.sub > 1 && total_tokens <= c.piece_len) c.sub = 1;  // one piece per sequence: nothing to fold
    return c;
}

long max_pieces(long total_tokens, int num_seqs, long piece_len) {
    return kda::max_pieces_of(total_tokens, num_seqs, piece_len);
}

kda::WorkspaceLayout layout_of(const kda::PlanChoice &c, long total_tokens, int num_seqs, int H, int dk,
                               int dv) {
    const long P = max_pieces(total_tokens, num_seqs, c.piece_len);
    const long Ps = c.sub > 1 ? max_pieces(total_tokens, num_seqs, c.piece_len / c.sub) : 0;
    return kda::workspace_layout(P, num_seqs, H, dk, dv, Ps);
}

}  // namespace

extern "C" {

const char *kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        default: return "KDA_ERR_UNKNOWN";
    }
}

size_t kda_chunk_fwd_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                                    int32_t dv, kda_dtype dtype) {
    if (total_tokens < 0 || num_seqs < 0 || H < 1 || !dim_ok(dk) || !dim_ok(dv)) return 0;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return 0;
    // enough for the plan of every kernel family the call may run (the
    // extended features and forced paths change the family)
    size_t total = layout_of(choose_plan(total_tokens, num_seqs, H, Path::chunk16), total_tokens, num_seqs, H,
                             dk, dv).total;
    if (dtype == KDA_DTYPE_BF16 && dk == 128 && dv == 128) {
        for (Path path : {Path::tc5, Path::chunk32})
            total = std::max(total, layout_of(choose_plan(total_tokens, num_seqs, H, path), total_tokens, num_seqs,
                                              H, dk, dv).total);
    }
    return total;
}

int kda_chunk_fwd_plan(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t *piece_len,
                       int32_t *max_pieces_out, int32_t *launches) {
    if (total_tokens < 0 || num_seqs < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    const int f = kda::prefill_impl_forced();
    const kda::PlanChoice c = choose_plan(total_tokens, num_seqs, H,
                                          f == 1 ? Path::chunk32 : (f == 3 || f == 4 ? Path::chunk16 : Path::tc5));
    const long L = c.piece_len;
    const long P = max_pieces(total_tokens, num_seqs, L);
    if (piece_len) *piece_len = (int32_t)L;
    if (max_pieces_out) *max_pieces_out = (int32_t)(P > 0x7fffffffL ? 0x7fffffffL : P);
    if (launches) *launches = num_seqs == 0 ? 0 : (total_tokens > L ? (c.sub > 1 ? 6 : 4) : 2);
    return KDA_OK;
}

int32_t kda_chunk_fwd_sub_pieces(int32_t total_tokens, int32_t num_seqs, int32_t H) {
    if (total_tokens < 0 || num_seqs < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    const int f = kda::prefill_impl_forced();
    if (f == 1 || f == 3 || f == 4) return 1;
    return choose_plan(total_tokens, num_seqs, H, Path::tc5).sub;
}

int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                     const void *gate, void *out, const int32_t *cu_seqlens,
                     const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens,
                     int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t flags,
                     const float *initial_state, float *final_state, int32_t snapshot_tokens,
                     float *snapshots, const int32_t *snapshot_offsets, void *workspace,
                     size_t workspace_bytes, kda_stream_t stream_) {
    cudaStream_t stream = (cudaStream_t)stream_;
    int rc = kda::check_prefill_sizes(num_seqs, total_tokens, H, dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (flags & ~kda::FLAG_ALL) return KDA_ERR_INVALID_ARG;
    if (snapshot_tokens < 0 || snapshot_tokens % 16 != 0) return KDA_ERR_INVALID_ARG;
    if (snapshot_tokens > 0) {
        if (!snapshots || !snapshot_offsets) return KDA_ERR_INVALID_ARG;
        if (!aligned(snapshots, 16) || !aligned(snapshot_offsets, 4)) return KDA_ERR_ALIGNMENT;
    }
    bool empty = false;
    rc = kda::check_prefill_buffers(q, k, v, g, beta, gate, out, cu_seqlens, cu_seqlens_host, num_seqs,
                                    total_tokens, H, dk, dv, dtype, initial_state, final_state, workspace,
                                    &empty);
    if (rc != KDA_OK || empty) return rc;
    // the plan with the real lengths, when known, never needs more workspace
    // than the length-blind one the workspace was sized for
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    const Path path = kda::chunk32_eligible(bf16, dk, dv, flags, snapshot_tokens)
                          ? Path::chunk32
                          : (kda::tc5_path(bf16, dk, dv, flags, snapshot_tokens) ? Path::tc5 : Path::chunk16);
    const kda::PlanChoice plan = choose_plan(total_tokens, num_seqs, H, path, cu_seqlens_host);
    const long L = plan.piece_len;
    const int sub = plan.sub;
    const long P_max = max_pieces(total_tokens, num_seqs, L);
    const long P_sub_max = sub > 1 ? max_pieces(total_tokens, num_seqs, L / sub) : 0;
    if (L > (1L << 30) || P_max > (1L << 30) || (long)H * P_max > (1L << 31) || (long)H * P_sub_max > (1L << 31))
        return KDA_ERR_UNSUPPORTED;
    const kda::WorkspaceLayout WL = kda::workspace_layout(P_max, num_seqs, H, dk, dv, P_sub_max);
    if (!workspace || workspace_bytes < WL.total) return KDA_ERR_WORKSPACE;

    char *ws = (char *)workspace;
    kda::PrefillParams p{};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.gate = gate; p.out = out;
    p.cu_seqlens = cu_seqlens;
    p.header = (const int32_t *)(ws + WL.off_header);
    p.err = (int32_t *)(ws + WL.off_header) + 2;
    p.seq_first = (const int32_t *)(ws + WL.off_seq_first);
    p.pieces = (const int4 *)(ws + WL.off_pieces);
    p.M = (float *)(ws + WL.off_M);
    p.Szero = (float *)(ws + WL.off_Szero);
    p.Sin = (float *)(ws + WL.off_Sin);
    p.initial_state = initial_state;
    p.final_state = final_state;
    p.num_seqs = num_seqs;
    p.H = H;
    p.P_max = (int)P_max;
    p.scale = scale;
    p.flags = flags;
    p.total_tokens = total_tokens;
    p.snap_tokens = snapshot_tokens;
    p.snapshots = snapshot_tokens > 0 ? snapshots : nullptr;
    p.snap_offsets = snapshot_tokens > 0 ? snapshot_offsets : nullptr;
    p.piece_len = (int)L;

    cudaError_t e = kda::launch_plan(cu_seqlens, num_seqs, total_tokens, (int)L, (int)P_max,
                                     (int32_t *)(ws + WL.off_header),
                                     (int32_t *)(ws + WL.off_seq_first),
                                     (int4 *)(ws + WL.off_pieces), stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    const bool multi = total_tokens > L;  // some sequence may have >1 piece
    // the summary pass over sub-pieces: its own plan tables and maps
    kda::PrefillParams ps = p;
    if (multi && sub > 1) {
        e = kda::launch_plan(cu_seqlens, num_seqs, total_tokens, (int)(L / sub), (int)P_sub_max,
                             (int32_t *)(ws + WL.off_header_sub), (int32_t *)(ws + WL.off_seq_first_sub),
                             (int4 *)(ws + WL.off_pieces_sub), stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        ps.seq_first = (const int32_t *)(ws + WL.off_seq_first_sub);
        ps.pieces = (const int4 *)(ws + WL.off_pieces_sub);
        ps.M = (float *)(ws + WL.off_M_sub);
        ps.Szero = (float *)(ws + WL.off_Szero_sub);
        ps.P_max = (int)P_sub_max;
        ps.piece_len = (int)(L / sub);
        ps.sub = sub;
    }
#ifdef KDA_CHECK_G
    // after the plan kernels, which clear the error word
    e = kda::launch_check_g(g, bf16, (long)total_tokens * H * dk, (flags & kda::FLAG_CLAMP_G) ? 1 : 0,
                            p.err, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
#endif
    if (multi) {
        e = kda::launch_prefill_chunks(ps, bf16, dk, dv, true, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        if (sub > 1) {
            kda::SubFoldParams f{};
            f.pieces = p.pieces;
            f.seq_first = p.seq_first;
            f.seq_first_sub = ps.seq_first;
            f.M_sub = ps.M;
            f.Z_sub = ps.Szero;
            f.M = p.M;
            f.Z = p.Szero;
            f.H = H;
            f.P_max = (int)P_max;
            f.P_sub_max = (int)P_sub_max;
            f.sub = sub;
            e = kda::launch_subfold_tc(f, p.err, stream);
            if (e != cudaSuccess) return KDA_ERR_CUDA;
        }
        e = kda::launch_scan(p, dk, dv, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    e = kda::launch_prefill_chunks(p, bf16, dk, dv, false, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

int kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  const void *gate, void *out, const int32_t *cu_seqlens,
                  const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens,
                  int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, float scale,
                  int32_t qk_l2norm, const float *initial_state, float *final_state,
                  void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    if (qk_l2norm != 0 && qk_l2norm != 1) return KDA_ERR_INVALID_ARG;
    return kda_chunk_fwd_ex(q, k, v, g, beta, gate, out, cu_seqlens, cu_seqlens_host, num_seqs,
                            total_tokens, H, dk, dv, dtype, scale, qk_l2norm, initial_state,
                            final_state, 0, nullptr, nullptr, workspace, workspace_bytes, stream);
}

int kda_chunk_fwd_check(const void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    if (!workspace || workspace_bytes < 3 * sizeof(int32_t)) return KDA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
    int32_t h[3];
    if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KDA_ERR_CUDA;
    return kda::decode_plan_header(h);
}

int kda_build_checks_g(void) {
#ifdef KDA_CHECK_G
    return 1;
#else
    return 0;
#endif
}

int kda_decode_step_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                       const void *gate, void *out, float *state, int32_t num_seqs, int32_t H,
                       int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t flags,
                       kda_stream_t stream) {
    if (num_seqs < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (flags & ~kda::FLAG_ALL) return KDA_ERR_INVALID_ARG;
    if (num_seqs == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !out || !state) return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const void *a16[] = {q, k, v, g, gate, out, state};
    for (const void *p : a16)
        if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    if (!aligned(beta, esz)) return KDA_ERR_ALIGNMENT;
    const long nh = (long)num_seqs * H;
    if (nh > 0x7fffffffL) return KDA_ERR_UNSUPPORTED;
    const cudaError_t e = kda::launch_decode(dtype == KDA_DTYPE_BF16, dk, dv, q, k, v, g, beta,
                                             gate, out, state, nh, scale, flags,
                                             (cudaStream_t)stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_decode_step(const void *q, const void *k, const void *v, const void *g, const void *beta,
                    const void *gate, void *out, float *state, int32_t num_seqs, int32_t H,
                    int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t qk_l2norm,
                    kda_stream_t stream) {
    if (qk_l2norm != 0 && qk_l2norm != 1) return KDA_ERR_INVALID_ARG;
    return kda_decode_step_ex(q, k, v, g, beta, gate, out, state, num_seqs, H, dk, dv, dtype, scale,
                              qk_l2norm, stream);
}

}  // extern "C"
