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
// held until the process exits.  It is placed when the library's device code
// is loaded on a device; under CUDA's lazy module loading that is the first
// call into this library there, so a caller that may not allocate later
// makes one call (kda_chunk_fwd_noalloc_check is enough) at start-up, before
// any stream capture.  Host code cannot use the array's name as a device
// address: every call looks the address up with cudaGetSymbolAddress on the
// current device (cheap once the code is loaded, and right again after the
// context has been reset).  Every call on a device uses the same array: calls
// that overlap on the GPU (different streams, or another host thread) race on
// it and must be serialised by the caller.  Nothing in the array has to start
// at zero: each call writes every entry it later reads.  The device-side
// error words of the last call sit in the array's first bytes and are read
// by kda_chunk_fwd_noalloc_check.
#include <cstdlib>

#include "../../include/kda.h"
#include "kda_args.h"
#include "kda_common.cuh"
#include "kda_prefill.cuh"

namespace kda {
cudaError_t launch_plan(const int32_t *cu, int num_seqs, int total_tokens, int piece_len, int P_max,
                        int32_t *header, int32_t *seq_first, int4 *pieces, cudaStream_t st);
cudaError_t launch_scan(const PrefillParams &p, int dk, int dv, cudaStream_t st);
cudaError_t launch_prefill_chunks(const PrefillParams &p, bool bf16, int dk, int dv,
                                  bool summaries, cudaStream_t st);
#ifdef KDA_CHECK_G
cudaError_t launch_check_g(const void *g, bool bf16, long n, int clamp, int32_t *err,
                           cudaStream_t st);
#endif
}  // namespace kda

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) unsigned char kda_noalloc_scratch[kScratchBytes];

// Device address of the scratch array on the current device.
int scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, kda_noalloc_scratch);
    if (e != cudaSuccess || !p) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    *out = p;
    return KDA_OK;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    return n;
}

// Scratch bytes the plan with piece length L needs: with a single piece per
// sequence only the plan table is used.
size_t scratch_need(long L, int num_seqs, int total_tokens, int H, int dk, int dv) {
    const long P = (long)num_seqs + ((long)total_tokens + L - 1) / L;
    const kda::WorkspaceLayout W = kda::workspace_layout(P, num_seqs, H, dk, dv);
    return total_tokens > L ? W.total : W.off_M;
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
    int rc = kda::check_prefill_sizes(num_seqs, total_tokens, H, dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (qk_l2norm != 0 && qk_l2norm != 1) return KDA_ERR_INVALID_ARG;
    bool empty = false;
    rc = kda::check_prefill_buffers(q, k, v, g, beta, gate, out, cu_seqlens, cu_seqlens_host, num_seqs,
                                    total_tokens, H, dk, dv, dtype, initial_state, final_state, nullptr,
                                    &empty);
    if (rc != KDA_OK || empty) return rc;

    // Piece length: the usual plan or, when its piece summaries do not fit in
    // the fixed scratch, the shortest multiple of the chunk length that fits
    // (the need only falls as pieces get longer).  Once a piece spans the
    // whole input no summaries are needed and only the plan table remains; if
    // even that does not fit, the sizes are beyond what this entry point
    // supports.
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    const bool c32 = kda::chunk32_eligible(bf16, dk, dv, qk_l2norm, 0);
    const kda::PlanModel pm = c32 ? kda::plan_model_chunk32(sm_count()) : kda::plan_model_chunk16(sm_count());
    const long C = pm.chunk;
    long L = kda::plan_piece_len(total_tokens, num_seqs, H, pm, cu_seqlens_host);
    if (scratch_need(L, num_seqs, total_tokens, H, dk, dv) > kScratchBytes) {
        long hi = ((long)total_tokens + C - 1) / C * C + C;  // one piece per sequence
        if (scratch_need(hi, num_seqs, total_tokens, H, dk, dv) > kScratchBytes)
            return KDA_ERR_WORKSPACE;  // sizes beyond the fixed scratch
        long lo = L;                   // does not fit
        while (hi - lo > C) {
            long mid = (lo + hi) / 2 / C * C;
            if (mid <= lo) mid = lo + C;
            if (scratch_need(mid, num_seqs, total_tokens, H, dk, dv) <= kScratchBytes) hi = mid;
            else lo = mid;
        }
        L = hi;
    }
    if (L > (1L << 30)) return KDA_ERR_UNSUPPORTED;
    const long P_max = (long)num_seqs + ((long)total_tokens + L - 1) / L;
    if (P_max > (1L << 30) || (long)H * P_max > (1L << 31)) return KDA_ERR_UNSUPPORTED;
    const kda::WorkspaceLayout WL = kda::workspace_layout(P_max, num_seqs, H, dk, dv);
    const bool summaries = total_tokens > L;

    void *scratch = nullptr;
    rc = scratch_address(&scratch);
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
    p.piece_len = (int)L;

    cudaError_t e = kda::launch_plan(cu_seqlens, num_seqs, total_tokens, (int)L, (int)P_max,
                                     (int32_t *)(ws + WL.off_header),
                                     (int32_t *)(ws + WL.off_seq_first),
                                     (int4 *)(ws + WL.off_pieces), stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
#ifdef KDA_CHECK_G
    // after the plan kernel, which clears the error word
    e = kda::launch_check_g(g, bf16, (long)total_tokens * H * dk, 0, p.err, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
#endif
    if (summaries) {
        e = kda::launch_prefill_chunks(p, bf16, dk, dv, true, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        e = kda::launch_scan(p, dk, dv, stream);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    e = kda::launch_prefill_chunks(p, bf16, dk, dv, false, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// Waits for `stream` and maps the error words of the last
// kda_chunk_fwd_noalloc call on the current device to a status (the same
// decoding as kda_chunk_fwd_check).  Copies 12 bytes from the scratch array to
// the host; allocates nothing.
extern "C" int kda_chunk_fwd_noalloc_check(kda_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
    int32_t h[3];
    if (cudaMemcpyFromSymbol(h, kda_noalloc_scratch, sizeof(h), 0, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    return kda::decode_plan_header(h);
}
