// kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// code inside a custom allocator or memory-pool callback, runtimes that own
// all device memory and hand out only fixed buffers, or plugins whose host
// application forbids allocation after start-up.  kda_chunk_fwd needs a
// workspace (the piece plan, and per piece and head a transition matrix and
// two states); here that workspace is a fixed array in device global memory
// that belongs to the library itself, so the caller passes only its inputs
// and outputs.
//
// The array (kScratchBytes) exists once per GPU that loads this code and is
// held until the process exits.  Host code cannot use its name as a device
// address, so the address is looked up with cudaGetSymbolAddress once per
// device, on the first call made while that device is current; make that
// first call before any stream capture.  Every call on a device uses the
// same array: calls that overlap on the GPU (different streams, or another
// host thread) race on it and must be serialised by the caller.  Nothing in
// the array has to start at zero: each call writes every entry it later
// reads.
#include <cstdlib>
#include <mutex>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {
cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st);
cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st);
cudaError_t launch_prefill_chunks(const PrefillParams &p, bool bf16, int dk, int dv,
                                  bool summaries, cudaStream_t st);
}  // namespace kda

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) unsigned char kda_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, kda_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return KDA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KDA_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128; }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    return n;
}

}  // namespace

extern "C" int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                                     const void *beta, const void *gate, void *out,
                                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                     int32_t num_seqs, int32_t total_tokens, int32_t H,
                                     int32_t dk, int32_t dv, kda_dtype dtype, float scale,
                                     int32_t qk_l2norm, const float *initial_state,
                                     float *final_state, kda_stream_t stream_) {
    cudaStream_t stream = (cudaStream_t)stream_;
    if (num_seqs < 0 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (qk_l2norm != 0 && qk_l2norm != 1) return KDA_ERR_INVALID_ARG;
    if (num_seqs == 0) return total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const void *a16[] = {q, k, v, g, gate, out, initial_state, final_state};
    for (const void *p : a16)
        if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    if (beta && !aligned(beta, esz)) return KDA_ERR_ALIGNMENT;
    if (!aligned(cu_seqlens, 4)) return KDA_ERR_ALIGNMENT;
    const size_t state_bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    if (initial_state && final_state && initial_state != final_state) {
        const char *a = (const char *)initial_state, *b = (const char *)final_state;
        if (a < b + state_bytes && b < a + state_bytes) return KDA_ERR_INVALID_ARG;
    }
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_tokens)
            return KDA_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    }

    // Piece length: the usual plan, lengthened until the piece summaries fit in the
    // fixed scratch array.  Once a piece spans the whole input no summaries
    // are needed and only the plan table remains; if even that does not fit,
    // the sizes are beyond what this entry point supports.
    long L = kda::plan_piece_len(total_tokens, num_seqs, H, sm_count(), cu_seqlens_host);
    const long L_all = ((long)total_tokens + 15) / 16 * 16 + 16;
    for (;;) {
        const long P = (long)num_seqs + ((long)total_tokens + L - 1) / L;
        const kda::WorkspaceLayout W = kda::workspace_layout(P, num_seqs, H, dk, dv);
        // with a single piece per sequence only the plan table is used
        const size_t need = total_tokens > L ? W.total : W.off_M;
        if (need <= kScratchBytes) break;
        if (L >= L_all) return KDA_ERR_WORKSPACE;  // sizes beyond the fixed scratch
        L = L * 2 < L_all ? L * 2 : L_all;
    }
    if (L > (1L << 30)) return KDA_ERR_UNSUPPORTED;
    const long P_max = (long)num_seqs + ((long)total_tokens + L - 1) / L;
    if (P_max > (1L << 30) || (long)H * P_max > (1L << 31)) return KDA_ERR_UNSUPPORTED;
    const kda::WorkspaceLayout WL = kda::workspace_layout(P_max, num_seqs, H, dk, dv);
    const bool summaries = total_tokens > L;

    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != KDA_OK) return rc;
    char *ws = (char *)scratch;

    kda::PrefillParams p{};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.gate = gate; p.out = out;
    p.cu_seqlens = cu_seqlens;
    p.header = (const int32_t *)(ws + WL.off_header);
    p.err = (int32_t *)(ws + WL.off_header) + 2;
    p.seq_first = (const int32_t *)(ws + WL.off_seq_first);
    p.pieces = (const int4 *)(ws + WL.off_pieces);
    p.M = summaries ? (float *)(ws + WL.off_M) : nullptr;
    p.Szero = summaries ? (float *)(ws + WL.off_Szero) : nullptr;
    p.Sin = summaries ? (float *)(ws + WL.off_Sin) : nullptr;
    p.initial_state = initial_state;
    p.final_state = final_state;
    p.num_seqs = num_seqs;
    p.H = H;
    p.P_max = (int)P_max;
    p.scale = scale;
    p.flags = qk_l2norm;
    p.snap_tokens = 0;
    p.snapshots = nullptr;
    p.snap_offsets = nullptr;
    p.total_tokens = total_tokens;

    const bool bf16 = dtype == KDA_DTYPE_BF16;
    cudaError_t e = kda::launch_plan(cu_seqlens, num_seqs, total_tokens, (int)L, (int)P_max,
                                     (int32_t *)(ws + WL.off_header),
                                     (int32_t *)(ws + WL.off_seq_first),
                                     (int4 *)(ws + WL.off_pieces), stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    if (summaries) {
        e = kda::launch_prefill_chunks(p, bf16, dk, dv, true, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        e = kda::launch_scan(p, dk, dv, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    e = kda::launch_prefill_chunks(p, bf16, dk, dv, false, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
