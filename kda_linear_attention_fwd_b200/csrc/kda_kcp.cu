// KDA context parallelism: the affine map of a token segment, and the
// composition of such maps.
//
// The tokens of a sequence segment act on an incoming state S as one affine
// map, S -> Mseg S + Sseg: Mseg (dk x dk) is how the segment transforms any
// incoming state and Sseg (dk x dv) is the state it produces from zero.  Both
// have a fixed size, independent of the segment's length, so a long sequence
// split over devices needs only these summaries to be exchanged; each device
// then folds the maps of the segments before its own into its incoming state
// (affta.cn K3 explainer, section "KDA 上下文并行，让上下文的交接变薄";
// prism.simon-ai.net, "从架构创新出发：K3的MoE与混合注意力设计", section
// "Linear Attention 的分层 Chunking 策略").
//
// kda_chunk_fwd_summary runs the chunk kernels' summary pass over every piece
// of every sequence and folds the pieces' maps in order.  kda_state_compose
// applies a list of maps to a state.  Both folds use one kernel: per (sequence,
// head, block of 16 state columns) it keeps the columns in shared memory and
// applies x <- M_i x (+ Z_i) for each map in turn, in fp32.
#include "kda_common.cuh"
#include "kda_prefill.cuh"
#include "kda.h"

#include <cstring>

namespace kda {

cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st);
cudaError_t launch_prefill_chunks(const PrefillParams &p, bool bf16, int dk, int dv, bool summaries,
                                  cudaStream_t st);

namespace {

constexpr int kCols = 16;

// Map i of sequence n, head h: index (first(n) + i * step) * H + h into M
// (dk x dk each) and Z (dk x nz each); first = seq_first (pieces) or null (n).
struct FoldParams {
    const float *M, *Z;
    const int32_t *first;  // per-sequence first map (null: first(n) = n)
    int step;              // maps between consecutive maps of one sequence
    int count;             // maps per sequence when first is null
    int N, H, nz;
    // summary mode: columns [0, dk) start as the identity and collect the
    // transition into outM; columns [dk, dk + nz) start at zero, add Z and
    // collect into outZ.  compose mode: nz columns start at sin (or zero), add
    // Z and collect into sout.
    bool summary;
    float *outM, *outZ;
    const float *sin;
    float *sout;
};

template <int DK>
__global__ void __launch_bounds__(256) fold_kernel(FoldParams f) {
    constexpr int RW = DK / 16;  // rows per thread
    extern __shared__ __align__(16) float Ms[];  // one map, DK * DK
    __shared__ float X[DK][kCols + 1];
    const int n = blockIdx.x, h = blockIdx.y;
    const int col = threadIdx.x % kCols, rg = threadIdx.x / kCols;
    const int c = blockIdx.z * kCols + col;  // column of [M | Z] (summary) or of the state
    const int H = f.H;
    const int first = f.first ? f.first[n] : n;
    const int cnt = f.first ? f.first[n + 1] - f.first[n] : f.count;
    const bool zcol = !f.summary || c >= DK;
    const int zc = f.summary ? c - DK : c;
    const size_t MS = (size_t)DK * DK, ZS = (size_t)DK * f.nz;

#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int i = rg * RW + r;
        float x0;
        if (f.summary) x0 = zcol ? 0.f : (i == c ? 1.f : 0.f);
        else x0 = f.sin ? f.sin[((size_t)n * H + h) * ZS + (size_t)i * f.nz + c] : 0.f;
        X[i][col] = x0;
    }
    for (int m = 0; m < cnt; ++m) {
        const size_t idx = (size_t)(first + (size_t)m * f.step) * H + h;
        const float4 *src = reinterpret_cast<const float4 *>(f.M + idx * MS);
        __syncthreads();  // the previous map's products are done
        for (int x = threadIdx.x; x < DK * DK / 4; x += 256) reinterpret_cast<float4 *>(Ms)[x] = src[x];
        __syncthreads();
        float acc[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            acc[r] = zcol ? f.Z[idx * ZS + (size_t)(rg * RW + r) * f.nz + zc] : 0.f;
#pragma unroll 4
        for (int kk = 0; kk < DK; ++kk) {
            const float xv = X[kk][col];
#pragma unroll
            for (int r = 0; r < RW; ++r) acc[r] += Ms[(rg * RW + r) * DK + kk] * xv;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RW; ++r) X[rg * RW + r][col] = acc[r];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int i = rg * RW + r;
        const size_t nh = (size_t)n * H + h;
        if (!f.summary) f.sout[nh * ZS + (size_t)i * f.nz + c] = X[i][col];
        else if (zcol) f.outZ[nh * ZS + (size_t)i * f.nz + zc] = X[i][col];
        else f.outM[nh * MS + (size_t)i * DK + c] = X[i][col];
    }
}

cudaError_t launch_fold(const FoldParams &f, int dk, cudaStream_t st) {
    const int cols = f.summary ? dk + f.nz : f.nz;
    const dim3 grid((unsigned)f.N, (unsigned)f.H, (unsigned)(cols / kCols));
    const int sm = dk * dk * (int)sizeof(float);
    cudaError_t e;
    if (dk == 128) {
        e = cudaFuncSetAttribute(fold_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        fold_kernel<128><<<grid, 256, sm, st>>>(f);
    } else {
        e = cudaFuncSetAttribute(fold_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        fold_kernel<64><<<grid, 256, sm, st>>>(f);
    }
    return cudaGetLastError();
}

bool dim_ok(int d) { return d == 64 || d == 128; }
bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace
}  // namespace kda

extern "C" {

int kda_chunk_fwd_summary(const void *k, const void *v, const void *g, const void *beta,
                          const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                          kda_dtype dtype, int32_t flags, float *transition, float *zero_state,
                          void *workspace, size_t workspace_bytes, kda_stream_t stream_) {
    using namespace kda;
    cudaStream_t stream = (cudaStream_t)stream_;
    if (num_seqs < 0 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (flags & ~FLAG_ALL) return KDA_ERR_INVALID_ARG;
    if (num_seqs == 0) return total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || !transition || !zero_state) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!k || !v || !g || !beta)) return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const void *a16[] = {k, v, g, transition, zero_state, workspace};
    for (const void *p : a16)
        if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    if (beta && !aligned(beta, esz)) return KDA_ERR_ALIGNMENT;
    if (!aligned(cu_seqlens, 4)) return KDA_ERR_ALIGNMENT;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_tokens)
            return KDA_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    }
    const PlanModel pm = chunk32_eligible(dtype == KDA_DTYPE_BF16, dk, dv, flags, 0)
                             ? plan_model_chunk32(sm_count())
                             : plan_model_chunk16(sm_count());
    const long L = plan_piece_len(total_tokens, num_seqs, H, pm, cu_seqlens_host);
    const long P_max = (long)num_seqs + ((long)total_tokens + L - 1) / L;
    if (P_max > (1L << 30) || (long)H * P_max > (1L << 31)) return KDA_ERR_UNSUPPORTED;
    const WorkspaceLayout WL = workspace_layout(P_max, num_seqs, H, dk, dv);
    if (!workspace || workspace_bytes < WL.total) return KDA_ERR_WORKSPACE;

    char *ws = (char *)workspace;
    PrefillParams p{};
    p.k = k; p.v = v; p.g = g; p.beta = beta;
    p.q = k;  // not read by the summary pass (no outputs); any valid tile source
    p.cu_seqlens = cu_seqlens;
    p.header = (const int32_t *)(ws + WL.off_header);
    p.err = (int32_t *)(ws + WL.off_header) + 2;
    p.seq_first = (const int32_t *)(ws + WL.off_seq_first);
    p.pieces = (const int4 *)(ws + WL.off_pieces);
    p.M = (float *)(ws + WL.off_M);
    p.Szero = (float *)(ws + WL.off_Szero);
    p.Sin = (float *)(ws + WL.off_Sin);
    p.num_seqs = num_seqs;
    p.H = H;
    p.P_max = (int)P_max;
    p.total_tokens = total_tokens;
    p.scale = 1.f;
    p.flags = flags;
    p.summarize_all = 1;
    p.piece_len = (int)L;

    cudaError_t e = launch_plan(cu_seqlens, num_seqs, total_tokens, (int)L, (int)P_max,
                                (int32_t *)(ws + WL.off_header), (int32_t *)(ws + WL.off_seq_first),
                                (int4 *)(ws + WL.off_pieces), stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    e = launch_prefill_chunks(p, dtype == KDA_DTYPE_BF16, dk, dv, true, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    FoldParams f{};
    f.M = p.M;
    f.Z = p.Szero;
    f.first = p.seq_first;
    f.step = 1;
    f.N = num_seqs;
    f.H = H;
    f.nz = dv;
    f.summary = true;
    f.outM = transition;
    f.outZ = zero_state;
    e = launch_fold(f, dk, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_state_compose(const float *transitions, const float *zero_states, int32_t count,
                      const float *state_in, float *state_out, int32_t num_seqs, int32_t H,
                      int32_t dk, int32_t dv, kda_stream_t stream) {
    using namespace kda;
    if (count < 0 || num_seqs < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return KDA_OK;
    if (!state_out || (count > 0 && (!transitions || !zero_states))) return KDA_ERR_INVALID_ARG;
    const void *a16[] = {transitions, zero_states, state_in, state_out};
    for (const void *p : a16)
        if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    const size_t bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    if (state_in && state_in != state_out) {
        const char *a = (const char *)state_in, *b = (const char *)state_out;
        if (a < b + bytes && b < a + bytes) return KDA_ERR_INVALID_ARG;
    }
    FoldParams f{};
    f.M = transitions;
    f.Z = zero_states;
    f.first = nullptr;
    f.step = num_seqs;
    f.count = count;
    f.N = num_seqs;
    f.H = H;
    f.nz = dv;
    f.summary = false;
    f.sin = state_in;
    f.sout = state_out;
    const cudaError_t e = launch_fold(f, dk, (cudaStream_t)stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
