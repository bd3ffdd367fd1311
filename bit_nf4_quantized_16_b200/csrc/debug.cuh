// Bounds checks of the QLORA_DEBUG build.  Every check names an index and the
// extent of the buffer it indexes; a failed check records its source line in
// this translation unit's debug word and the access is skipped, so a bad index
// becomes a status read back on the host (qlora_debug_bounds) instead of a
// memory fault.  In the ordinary build QLORA_IN(i, n) is the constant true and
// costs nothing.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

// Host registry of the per-translation-unit debug words (api.cu).  A reader
// returns the recorded line (0 if none, -1 on a CUDA error) and clears it.
typedef int (*BoundsReader)();
void register_bounds_reader(BoundsReader reader, const char *unit);

#ifdef QLORA_DEBUG
namespace {
__device__ int g_bounds_line;   // first source line whose check failed, 0 if none

__device__ __forceinline__ bool in_bounds(int64_t i, int64_t n, int line)
{
    if (i >= 0 && i < n) return true;
    atomicCAS(&g_bounds_line, 0, line);
    return false;
}

int read_bounds_line()
{
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_bounds_line, sizeof(int)) != cudaSuccess) return -1;
    if (v && cudaMemcpyToSymbol(g_bounds_line, &zero, sizeof(int)) != cudaSuccess) return -1;
    return v;
}

struct BoundsRegistration {
    BoundsRegistration() { register_bounds_reader(&read_bounds_line, __BASE_FILE__); }
} g_bounds_registration;
}  // namespace
#define QLORA_IN(i, n) ::qlora::in_bounds((int64_t)(i), (int64_t)(n), __LINE__)
#else
#define QLORA_IN(i, n) true
#endif

}  // namespace qlora
