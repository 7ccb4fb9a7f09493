// Test helper (compiled by tests/test_gpu_speculation.py): a kernel that lets the next launch in the
// stream start at once (programmatic dependent launch) and only then, after a bounded sleep,
// overwrites a lens array -- the preceding grid that a decode's speculative set-up must survive.
#include <cuda_runtime.h>

extern "C" __global__ void k_late_lens(int *lens, const int *new_lens, int n, unsigned sleep_us) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (unsigned i = 0; i < sleep_us; ++i) __nanosleep(1000);
    for (int i = threadIdx.x; i < n; i += blockDim.x) lens[i] = new_lens[i];
}

extern "C" int launch_late_lens(int *lens, const int *new_lens, int n, unsigned sleep_us, void *stream) {
    k_late_lens<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(lens, new_lens, n, sleep_us);
    return static_cast<int>(cudaGetLastError());
}
