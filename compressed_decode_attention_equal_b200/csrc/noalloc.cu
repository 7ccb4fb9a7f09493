// skv_decode_attn_noalloc: compressed decode attention for callers that cannot allocate device
// memory -- for example code running inside a CUDA graph it does not own, a plugin handed only its
// input and output buffers by a host framework, or an embedded runtime whose allocator is fixed at
// start-up. Instead of a caller-provided workspace it uses one scratch array that the library
// itself defines at file scope, so loading the library reserves it once on every GPU that loads
// the module and it stays reserved until the process exits. The kernel is the same one
// skv_decode_attn launches; only where its scratch lives differs.
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

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

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
    // the same argument rules as skv_decode_attn
    if (B < 1 || R < 1 || Hq < 1 || Hkv < 1 || max_pages < 1) return SKV_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || (d != 64 && d != 128) || (dtype != SKV_BF16 && dtype != SKV_F32))
        return SKV_ERR_UNSUPPORTED;
    if (!q || !out || !lse || !pool || !page_table || !lens) return SKV_ERR_INVALID_ARG;
    if (!pool->pages || pool->num_pages < 0) return SKV_ERR_INVALID_ARG;
    const auto al = [](const void *p, uintptr_t m) { return (reinterpret_cast<uintptr_t>(p) & (m - 1)) == 0; };
    if (!al(pool->pages, 16) || !al(q, 16) || !al(out, 16) || !al(lse, 4)) return SKV_ERR_INVALID_ARG;
    const int64_t rows = static_cast<int64_t>(R) * (Hq / Hkv);
    if (rows > (1 << 20) || static_cast<int64_t>(max_pages) * kPageNodes > INT32_MAX / 2) return SKV_ERR_UNSUPPORTED;
    DecodeArgs a{};
    a.rows = static_cast<int>(rows);
    a.row_passes = (a.rows + kRowsPerPass - 1) / kRowsPerPass;
    a.pass_rows = a.rows > kRowsPerPass ? kRowsPerPass : ((a.rows + 7) / 8) * 8;
    const int64_t nv = static_cast<int64_t>(B) * Hkv * a.row_passes;
    if (nv > kMaxVUnits || static_cast<int64_t>(B) * Hkv * max_pages * a.row_passes > INT32_MAX / 2)
        return SKV_ERR_UNSUPPORTED;
    a.n_vunits = static_cast<int>(nv);
    a.q = q;
    a.pages = static_cast<const uint8_t *>(pool->pages);
    a.num_pages = pool->num_pages;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.lens = lens;
    a.out = out;
    a.lse = lse;
    a.B = B;
    a.R = R;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.d = d;
    a.dtype = dtype;

    // carve the static scratch for the grid the launcher will use (bf16 caches keep split partials)
    int ncta = 0;
    if (dtype == SKV_BF16 && decode_split_ctas(a, &ncta) != cudaSuccess) return SKV_ERR_CUDA;
    const size_t counters = kWsHeader;
    const size_t part_v = counters + round256(static_cast<size_t>(nv) * 4);
    const size_t part_l = part_v + round256(static_cast<size_t>(ncta) * 2 * a.pass_rows * d * 4);
    const size_t total = part_l + round256(static_cast<size_t>(ncta) * 2 * a.pass_rows * 4);
    if (total > SKV_NOALLOC_SCRATCH_BYTES) return SKV_ERR_WORKSPACE;   // beyond the built-in maximum

    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return SKV_ERR_CUDA;
    uint8_t *base = static_cast<uint8_t *>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the flags and the completion counters must
    // start at zero (the partials are always written before they are read)
    if (cudaMemsetAsync(base, 0, part_v, s) != cudaSuccess) return SKV_ERR_CUDA;
    a.flags = reinterpret_cast<uint32_t *>(base);
    a.counters = reinterpret_cast<int32_t *>(base + counters);
    a.part_v = reinterpret_cast<float *>(base + part_v);
    a.part_l = reinterpret_cast<float *>(base + part_l);
    a.ncta = ncta;
    return launch_decode(a, s) == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}
