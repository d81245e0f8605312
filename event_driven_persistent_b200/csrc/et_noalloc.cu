// et_run_splitk_noalloc: the split-K megakernel with its whole workspace in
// a file-scope device array, for callers that must not allocate device
// memory.  See include/et.h for the contract.
#include <cuda_runtime.h>

#include <cstring>

#include "et_params.h"

namespace et {
cudaError_t splitk_setup(int* max_blocks_per_sm);
cudaError_t launch_splitk(const SplitKParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
}  // namespace et

using namespace et;

namespace {

// Limits of the allocation-free variant.
constexpr int kNaMaxRows = 65536;  // rows of A
constexpr int kNaCols = 128;       // columns of A (fixed)
constexpr int kNaChunk = 32;       // K chunk (fixed)
constexpr int kNaTileRows = 32;    // rows per task (fixed)
constexpr int kNaMaxTiles = kNaMaxRows / kNaTileRows;
constexpr int kNaChunks = kNaCols / kNaChunk;
constexpr int kNaFetch = 4;                                  // tasks per queue pop
constexpr int kNaMaxCtas = 256;                              // upper bound on SMs
constexpr int kNaCtr = kCtrFirstEvent + kNaMaxTiles + 1;     // one counter set
constexpr int kNaQueue = kNaMaxTiles * kNaChunks + kNaMaxTiles + kNaMaxCtas * kNaFetch + 64;

// Layout of the array: control block | counter set 0 | counter set 1 |
// ready-queue slots | one trace record (unused).
constexpr size_t kOffCtl = 0;
constexpr size_t kOffCtr0 = 256;
constexpr size_t kOffCtr1 = kOffCtr0 + ((kNaCtr * sizeof(int) + 255) / 256) * 256;
constexpr size_t kOffQueue = kOffCtr1 + ((kNaCtr * sizeof(int) + 255) / 256) * 256;
constexpr size_t kOffTrace = kOffQueue + ((kNaQueue * sizeof(unsigned long long) + 255) / 256) * 256;
constexpr size_t kNaBytes = kOffTrace + 256;
static_assert(sizeof(Ctl) <= 256, "control block");

// The workspace.  Every GPU that loads this library holds it (108,032 B)
// until the process exits.  In host code `g_na_scratch` names a host-side
// stand-in, not device memory: only the address from cudaGetSymbolAddress
// may be handed to a kernel.
static __device__ __align__(256) unsigned char g_na_scratch[kNaBytes];

constexpr int kNaMaxDevices = 64;
struct NaDevice {
    unsigned char* base = nullptr;  // device address of g_na_scratch on this device
    int n_ctas = 0;
    uint32_t epoch = 0;
};
NaDevice g_na[kNaMaxDevices];

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15) == 0; }

}  // namespace

extern "C" et_status et_run_splitk_noalloc(const float* A, int n_rows, float* Bpart, float* C, void* stream) {
    if (n_rows < 0 || n_rows > kNaMaxRows) return ET_ERR_INVALID;
    if (n_rows == 0) return ET_OK;
    if (!aligned16(A) || !aligned16(Bpart) || !aligned16(C)) return ET_ERR_INVALID;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) return ET_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    NaDevice& nd = g_na[dev];
    if (!nd.base) {
        // first call on this device: resolve the array's device address,
        // opt the kernel in to its shared memory, clear the workspace
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ET_ERR_CUDA;
        if (prop.major != 10) return ET_ERR_UNSUPPORTED;
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_na_scratch) != cudaSuccess || !ptr) return ET_ERR_CUDA;
        int mb = 0;
        if (splitk_setup(&mb) != cudaSuccess || mb < 1) return ET_ERR_UNSUPPORTED;
        if (cudaMemsetAsync(ptr, 0, kNaBytes, s) != cudaSuccess) return ET_ERR_CUDA;
        nd.n_ctas = prop.multiProcessorCount < kNaMaxCtas ? prop.multiProcessorCount : kNaMaxCtas;
        nd.base = static_cast<unsigned char*>(ptr);
    }
    SplitKParams p;
    memset(&p, 0, sizeof(p));
    p.A = A;
    p.Bp = Bpart;
    p.C = C;
    p.rows = n_rows;
    p.cols = kNaCols;
    p.chunk = kNaChunk;
    p.tile_rows = kNaTileRows;
    p.n_tiles = (n_rows + kNaTileRows - 1) / kNaTileRows;
    p.n_chunks = kNaChunks;
    p.ev_base = kCtrFirstEvent;
    p.ev_all = kCtrFirstEvent + kNaMaxTiles;
    RunArgs ra;
    memset(&ra, 0, sizeof(ra));
    // The call number selects the counter set; it is committed only after a
    // successful launch, so a launch that failed leaves the next call on the
    // set the previous call cleared.
    const uint32_t ep = nd.epoch + 1;
    int* ctr0 = reinterpret_cast<int*>(nd.base + kOffCtr0);
    int* ctr1 = reinterpret_cast<int*>(nd.base + kOffCtr1);
    ra.ctl = reinterpret_cast<Ctl*>(nd.base + kOffCtl);
    ra.ctr = (ep & 1) ? ctr1 : ctr0;       // zero at entry (cleared by the previous call)
    ra.ctr_next = (ep & 1) ? ctr0 : ctr1;  // cleared during this call
    ra.n_ctr = kNaCtr;
    ra.qslots = reinterpret_cast<unsigned long long*>(nd.base + kOffQueue);
    ra.qcap = kNaQueue;
    ra.epoch = ep;
    ra.n_init = p.n_tiles * p.n_chunks;
    ra.total_static = ra.n_init + p.n_tiles;
    ra.dynamic = 1;
    ra.fetch_batch = kNaFetch;
    ra.trace = reinterpret_cast<TraceRec*>(nd.base + kOffTrace);
    ra.trace_cap = 1;
    ra.timeout_ns = 1000000000ull;
    if (launch_splitk(p, ra, nd.n_ctas, s) != cudaSuccess) return ET_ERR_CUDA;  // nothing was enqueued
    nd.epoch = ep;
    // Synchronous: read the device status of this call, and after a device
    // error clear the workspace so the next call starts clean.
    Ctl h;
    if (cudaMemcpyAsync(&h, ra.ctl, sizeof(Ctl), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ET_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ET_ERR_CUDA;
    if (h.status != 0) {
        if (cudaMemsetAsync(nd.base, 0, kNaBytes, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
            return ET_ERR_CUDA;
        return (et_status)h.status;
    }
    return ET_OK;
}
