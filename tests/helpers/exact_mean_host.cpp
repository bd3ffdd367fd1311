// Host build of the library's exactly-rounded-mean routine, for CPU tests only:
// buckets the values the way the quantize kernel does, then calls the same
// header-only code the kernel uses.
#include <stdint.h>
#include <string.h>
#include "../../bit_nf4_quantized_16_b200/csrc/exact_mean.cuh"

extern "C" uint32_t host_exact_mean_bits(const float *v, int64_t n)
{
    unsigned long long bucket[256];
    memset(bucket, 0, sizeof(bucket));
    for (int64_t i = 0; i < n; i++) {
        uint32_t bits, b, s;
        memcpy(&bits, &v[i], 4);
        qlora::exact_mean_split(bits, &b, &s);
        bucket[b] += s;
    }
    return qlora::exact_mean_bits(bucket, (uint64_t)n);
}
