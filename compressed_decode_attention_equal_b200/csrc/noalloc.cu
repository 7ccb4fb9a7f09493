// skv_decode_attn_noalloc: compressed decode attention for callers that cannot allocate device
// memory -- for example a plugin that a host framework hands only its input and output buffers, a
// runtime whose device allocator is fixed when it starts, or code on a latency-critical path where
// a cudaMalloc (which may synchronise the device) is not allowed. Instead of a caller-provided
// workspace it uses one scratch array that the library itself defines at file scope, so loading
// the library reserves it once on every GPU that loads the module and it stays reserved until the
// process exits. The arguments are checked and planned by the same code as skv_decode_attn, and
// the kernel is the same one; only where its scratch lives differs.
#include <cstring>
#include <mutex>
#include <vector>

#include "skv_common.cuh"
#include "skv_internal.h"

using namespace skv;

namespace {

// Scratch of the no-allocation entry point: device error flags, per-unit completion counters and
// split partials. Every call on a device shares it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SKV_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device. In host code the array's name is only a host
// stand-in, so kernels must be given the address cudaGetSymbolAddress returns on that device.
std::mutex g_mu;
std::vector<std::pair<int, void *>> g_addr;

cudaError_t scratch_address(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    for (const auto &p : g_addr)
        if (p.first == dev) {
            *ptr = p.second;
            return cudaSuccess;
        }
    void *addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);   // with `dev` current
    if (e != cudaSuccess) return e;
    g_addr.emplace_back(dev, addr);
    *ptr = addr;
    return cudaSuccess;
}

}  // namespace

extern "C" skv_status skv_decode_attn_noalloc(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                                              const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                                              const int32_t *lens, void *out, float *lse, void *stream) {
    DecodePlan plan;
    DecodeArgs a;
    const skv_status st = decode_args(q, dtype, B, R, Hq, Hkv, d, pool, page_table, max_pages, lens, out, lse,
                                      SKV_CLOSURE_SCALAR, &plan, &a);
    if (st != SKV_OK) return st;

    // carve the static scratch for the grid the launcher will use (bf16 caches keep split partials;
    // the launcher sizes the same grid from the same cached occupancy query)
    int ncta = 0;
    if (dtype == SKV_BF16 && decode_split_ctas(a, &ncta) != cudaSuccess) return SKV_ERR_CUDA;
    const DecodeLayout lay = decode_layout(dtype, d, plan, ncta);
    if (lay.total > SKV_NOALLOC_SCRATCH_BYTES) return SKV_ERR_WORKSPACE;   // beyond the built-in maximum

    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return SKV_ERR_CUDA;
    uint8_t *base = static_cast<uint8_t *>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the flags and the completion counters must
    // start at zero (the partials are always written before they are read)
    if (cudaMemsetAsync(base, 0, lay.part_v, s) != cudaSuccess) return SKV_ERR_CUDA;
    a.flags = reinterpret_cast<uint32_t *>(base);
    a.counters = reinterpret_cast<int32_t *>(base + lay.counters);
    a.part_v = reinterpret_cast<float *>(base + lay.part_v);
    a.part_l = reinterpret_cast<float *>(base + lay.part_l);
    return launch_decode(a, s) == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}
