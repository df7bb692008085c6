// plan_noalloc.cu - moe_plan_noalloc: the routing and planning steps of
// moe_plan for callers that cannot allocate device memory.
//
// Some callers are handed only their input and output buffers and may not
// allocate anything themselves: a plugin running inside another framework's
// execution engine that offers no workspace, or a serving loop whose device
// memory is reserved up front by its own pool allocator, where cudaMalloc
// could fail once the pool owns the free memory and can synchronise the
// device in the middle of a latency-critical step. For them this file keeps
// the planner's scratch (per-chunk histograms and offsets, the piece and
// block tables, the block schedule, the padded-row map) in one static device
// array, so a call needs no workspace and allocates nothing.
//
// The array's name is only a host-side stand-in in host code; a kernel given
// it would fault, or on systems where the GPU can reach host memory would
// silently use the wrong memory. Every call therefore looks up the array's
// device address on the current device with cudaGetSymbolAddress (a lookup,
// no allocation) and hands that address to the kernels. Looking it up on
// every call rather than once keeps the address right after a
// cudaDeviceReset, which reloads the library's module and may move the array.
// The first lookup on a device loads the module there, so that first call
// belongs before any stream capture.
#include "common.cuh"

namespace {

// Largest scratch one call can use; every GPU that loads the library keeps
// this much device memory reserved until the process exits.
constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;

}  // namespace

static __device__ __align__(256) unsigned char g_plan_scratch[kScratchBytes];

namespace {

// The device address of g_plan_scratch on the current device.
cudaError_t scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_plan_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_plan_noalloc(const moe_config* cfg, const float* logits, int32_t* topk_idx,
                                       float* topk_w, int32_t* counts, int32_t* row_of, uint32_t* header,
                                       moe_stream_t stream) {
    using namespace moe;
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!logits || !topk_idx || !topk_w || !counts || !row_of || !header) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(counts) ||
        !aligned16(row_of) || !aligned16(header))
        return MOE_ERR_INVALID_ARG;
    // The scratch holds the plan part of a workspace; its header and row map
    // are replaced by the caller's buffers.
    const WsLayout L = make_layout(s);
    if ((size_t)L.plan_end > kScratchBytes) return MOE_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    WsPtrs P = ws_ptrs(scratch, L);
    P.header = header;
    P.row_of = row_of;
    // Nothing in the scratch has to start at zero: every word a kernel reads
    // is written earlier in this same call (chunk histograms and flags by the
    // top-k kernel, offsets, pieces, blocks and padding rows by the planner).
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_topk_hist(s, logits, topk_idx, topk_w, P, st);
    if (e == cudaSuccess) e = launch_plan(s, counts, P, st);
    if (e == cudaSuccess) e = launch_row_maps(s, topk_idx, P, st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
