// Host-side entry points that launch nothing: the NF4 codebook, status
// strings, device queries and the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <atomic>
#include <mutex>
#include <vector>
#include <string.h>

#include "common.cuh"
#include "debug.cuh"

namespace qlora {

// One error word per device; kernels receive its address as a parameter.
static __device__ int g_device_error = 0;

namespace {
int *g_error_ptr[kMaxDevices] = {};
DeviceInfo g_info[kMaxDevices];
bool g_info_ok[kMaxDevices] = {};
std::mutex g_mutex;
}  // namespace

qlora_status device_info(DeviceInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_info_ok[dev]) {
        DeviceInfo d;
        d.device = dev;
        int v = 0;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QLORA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return QLORA_ERR_CUDA;
        d.smem_optin = (size_t)v;
        g_info[dev] = d;
        g_info_ok[dev] = true;
    }
    *out = g_info[dev];
    // the kernels are built for sm_100a only
    if (out->major != 10) return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

// ---- tensor maps (TMA descriptors) ---------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

qlora_status make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn) return QLORA_ERR_CUDA;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

int *device_error_word()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_error_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_error_ptr[dev] = static_cast<int *>(p);
    }
    return g_error_ptr[dev];
}

qlora_status check_weight(const qlora_nf4_weight *w)
{
    if (!w) return QLORA_ERR_INVALID_ARG;
    if (w->rows <= 0 || w->cols <= 0 || w->cols % QLORA_BLOCK != 0) return QLORA_ERR_SHAPE;
    if (w->rows > ((int64_t)1 << 40) / w->cols) return QLORA_ERR_SHAPE;   // rows * cols stays far from overflow
    if (!w->packed || !w->code2 || !w->c2 || !w->mean) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(w->packed) || !aligned16(w->code2) || !aligned16(w->c2) || !aligned16(w->mean))
        return QLORA_ERR_ALIGNMENT;
    int zeros = 0;
    for (int j = 0; j < 16; j++) {
        if (!isfinite(w->codebook[j])) return QLORA_ERR_INVALID_ARG;
        if (j && !(w->codebook[j - 1] < w->codebook[j])) return QLORA_ERR_INVALID_ARG;
        zeros += w->codebook[j] == 0.0f;
    }
    if (zeros != 1) return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

// ---- normal quantile function -----------------------------------------------------
//
// Algorithm AS 241 (M. J. Wichura, "The percentage points of the normal
// distribution", Applied Statistics 37 (1988) 477-484), routine PPND16:
// rational approximations in q = p - 1/2 for the central region |q| <= 0.425
// and in t = sqrt(-ln min(p, 1-p)) for the tails, accurate to about 1e-16.
static double ppnd16(double p)
{
    static const double a[8] = {3.3871328727963666080e0, 1.3314166789178437745e+2, 1.9715909503065514427e+3,
                                1.3731693765509461125e+4, 4.5921953931549871457e+4, 6.7265770927008700853e+4,
                                3.3430575583588128105e+4, 2.5090809287301226727e+3};
    static const double b[8] = {1.0, 4.2313330701600911252e+1, 6.8718700749205790830e+2, 5.3941960214247511077e+3,
                                2.1213794301586595867e+4, 3.9307895800092710610e+4, 2.8729085735721942674e+4,
                                5.2264952788528545610e+3};
    static const double c[8] = {1.42343711074968357734e0, 4.63033784615654529590e0, 5.76949722146069140550e0,
                                3.64784832476320460504e0, 1.27045825245236838258e0, 2.41780725177450611770e-1,
                                2.27238449892691845833e-2, 7.74545014278341407640e-4};
    static const double d[8] = {1.0, 2.05319162663775882187e0, 1.67638483018380384940e0, 6.89767334985100004550e-1,
                                1.48103976427480074590e-1, 1.51986665636164571966e-2, 5.47593808499534494600e-4,
                                1.05075007164441684324e-9};
    static const double e[8] = {6.65790464350110377720e0, 5.46378491116411436990e0, 1.78482653991729133580e0,
                                2.96560571828504891230e-1, 2.65321895265761230930e-2, 1.24266094738807843860e-3,
                                2.71155556874348757815e-5, 2.01033439929228813265e-7};
    static const double f[8] = {1.0, 5.99832206555887937690e-1, 1.36929880922735805310e-1, 1.48753612908506148525e-2,
                                7.86869131145613259100e-4, 1.84631831751005468180e-5, 1.42151175831644588870e-7,
                                2.04426310338993978564e-15};
    auto poly = [](const double *k, double x) {
        double s = k[7];
        for (int i = 6; i >= 0; i--) s = s * x + k[i];
        return s;
    };
    double q = p - 0.5;
    if (fabs(q) <= 0.425) {
        double r = 0.180625 - q * q;
        return q * poly(a, r) / poly(b, r);
    }
    double r = q < 0 ? p : 1.0 - p;
    r = sqrt(-log(r));
    double x;
    if (r <= 5.0) {
        r -= 1.6;
        x = poly(c, r) / poly(d, r);
    } else {
        r -= 5.0;
        x = poly(e, r) / poly(f, r);
    }
    return q < 0 ? -x : x;
}

}  // namespace qlora

using namespace qlora;

// NF-k construction ("QLoRA: Efficient Finetuning of Quantized LLMs", section
// "Method", paragraph "4-bit NormalFloat Quantization"): 2^(k-1)+1 quantiles
// for the positive part and 2^(k-1) for the negative part, probabilities
// equally spaced from 1 - delta to 1/2, union without the duplicate zero,
// normalized by the largest magnitude into [-1, 1]; v receives the 2^k
// values ascending.
static void nfk_values(int k, double delta, double *v)
{
    const double hi = 1.0 - delta;
    const double top = ppnd16(hi);
    const int npos = (1 << (k - 1)) + 1, nneg = 1 << (k - 1);
    int n = 0;
    for (int i = 0; i < npos; i++) {     // positive part, zero included
        double p = i < npos - 1 ? hi + (0.5 - hi) * i / (double)(npos - 1) : 0.5;
        v[n++] = (i < npos - 1 ? ppnd16(p) : 0.0) / top;
    }
    for (int i = 0; i < nneg - 1; i++) {  // negative part; its zero is the dropped duplicate
        double p = hi + (0.5 - hi) * i / (double)(nneg - 1);
        v[n++] = -ppnd16(p) / top;
    }
    for (int i = 1; i < n; i++)           // ascending order
        for (int j = i; j > 0 && v[j - 1] > v[j]; j--) {
            double t = v[j];
            v[j] = v[j - 1];
            v[j - 1] = t;
        }
}

extern "C" qlora_status qlora_build_nf4_codebook(double delta, float codebook_out[16])
{
    if (!codebook_out) return QLORA_ERR_INVALID_ARG;
    if (delta <= 0.0) delta = 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    if (!(delta < 0.5)) return QLORA_ERR_INVALID_ARG;
    double v[16];
    nfk_values(4, delta, v);
    for (int i = 0; i < 16; i++) codebook_out[i] = (float)v[i];
    return QLORA_OK;
}

// NF-k for k = 2, 3, 4 in the 16-entry table of the 4-bit codec: the 2^k
// values, and 16 - 2^k padding values beyond +-1 (half at -1 - i/4 below,
// half at 1 + i/4 above), never the nearest value of anything in [-1, 1].
// Default delta: 1/2 (1/(2 * 2^k) + 1/(2 (2^k - 1))).
extern "C" qlora_status qlora_build_nfk_codebook(int k, double delta, float codebook_out[16])
{
    if (!codebook_out || k < 2 || k > 4) return QLORA_ERR_INVALID_ARG;
    const int n = 1 << k;
    if (delta <= 0.0) delta = 0.5 * (1.0 / (2.0 * n) + 1.0 / (2.0 * (n - 1)));
    if (!(delta < 0.5)) return QLORA_ERR_INVALID_ARG;
    double v[16];
    nfk_values(k, delta, v);
    const int half = (16 - n) / 2;
    for (int i = 0; i < half; i++) codebook_out[i] = (float)(-1.0 - (half - i) / 4.0);
    for (int i = 0; i < n; i++) codebook_out[half + i] = (float)v[i];
    for (int i = 0; i < half; i++) codebook_out[half + n + i] = (float)(1.0 + (i + 1) / 4.0);
    return QLORA_OK;
}

// Int4 as an absmax code ("QLoRA: Efficient Finetuning of Quantized LLMs",
// section "Introduction", item (1), compares NF4 with 4-bit integers without
// defining them): the 16 two's-complement integers -8 .. 7 divided by 7, so
// that +-7 carry the block's absmax.  -8/7 lies beyond -1 and is never the
// nearest value to a scaled element.
extern "C" qlora_status qlora_build_int4_codebook(float codebook_out[16])
{
    if (!codebook_out) return QLORA_ERR_INVALID_ARG;
    for (int j = 0; j < 16; j++) codebook_out[j] = (float)((double)(j - 8) / 7.0);
    return QLORA_OK;
}

// 4-bit float as an absmax code ("QLoRA: Efficient Finetuning of Quantized
// LLMs", section "Introduction", item (1), compares NF4 with 4-bit floats
// without defining them): the values of the E2M1 element type (sign, two
// exponent bits with bias 1, one mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2,
// 3, 4, 6) over the largest magnitude 6.  +0 and -0 are one table value, so
// the sixteenth entry is -8/6 (one exponent step beyond 6), below -1 and never
// the nearest value to a scaled element.
extern "C" qlora_status qlora_build_fp4_codebook(float codebook_out[16])
{
    if (!codebook_out) return QLORA_ERR_INVALID_ARG;
    static const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    codebook_out[0] = (float)(-8.0 / 6.0);
    for (int i = 0; i < 7; i++) codebook_out[1 + i] = (float)(-mags[7 - i] / 6.0);   // -1 .. -1/12
    for (int i = 0; i < 8; i++) codebook_out[8 + i] = (float)(mags[i] / 6.0);        // 0 .. 1
    return QLORA_OK;
}

extern "C" const char *qlora_status_string(qlora_status status)
{
    switch (status) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE";
    case QLORA_ERR_ALIGNMENT: return "QLORA_ERR_ALIGNMENT";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED";
    case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT";
    }
    return "QLORA_ERR_UNKNOWN";
}

extern "C" qlora_status qlora_check_device_error(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (v == kDevOk) return QLORA_OK;
    int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    return v == kDevTimeout ? QLORA_ERR_TIMEOUT : QLORA_ERR_CUDA;
}

// ---- failure-detection test hook -----------------------------------------------------

namespace qlora {
namespace {
std::mutex g_stall_mutex;
int g_stall_kind = -1;
uint64_t g_stall_ns = 0;
}  // namespace

bool take_stall_injection(int kind, uint64_t *timeout_ns)
{
    std::lock_guard<std::mutex> lock(g_stall_mutex);
    if (g_stall_kind != kind) return false;
    g_stall_kind = -1;
    *timeout_ns = g_stall_ns;
    return true;
}
}  // namespace qlora

extern "C" qlora_status qlora_debug_inject_stall(int kind, uint64_t timeout_ns)
{
    std::lock_guard<std::mutex> lock(g_stall_mutex);
    if (kind == -1) {
        g_stall_kind = -1;
        return QLORA_OK;
    }
    if (kind != QLORA_KERNEL_QUANTIZE && kind != QLORA_KERNEL_FWD_FUSED && kind != QLORA_KERNEL_BWD_FUSED)
        return QLORA_ERR_INVALID_ARG;
    if (timeout_ns < 1000ull || timeout_ns > 2000000000ull) return QLORA_ERR_INVALID_ARG;
    g_stall_kind = kind;
    g_stall_ns = timeout_ns;
    return QLORA_OK;
}

// ---- bounds-checked build ------------------------------------------------------------

namespace qlora {
namespace {
struct BoundsRegistry {
    std::mutex mu;
    std::vector<std::pair<BoundsReader, const char *>> readers;
};
BoundsRegistry &bounds_registry()
{
    static BoundsRegistry r;
    return r;
}
}  // namespace

void register_bounds_reader(BoundsReader reader, const char *unit)
{
    BoundsRegistry &r = bounds_registry();
    std::lock_guard<std::mutex> lock(r.mu);
    r.readers.emplace_back(reader, unit);
}
}  // namespace qlora

#ifdef QLORA_DEBUG
namespace qlora {
namespace {
// Evaluates one check whose index is past its extent; touches no memory.
__global__ void bounds_selftest_kernel(int64_t i, int64_t n, int *sink)
{
    if (!QLORA_IN(i, n) && sink) *sink = 1;
}
}  // namespace
}  // namespace qlora
#endif

extern "C" qlora_status qlora_debug_bounds_selftest(void)
{
#ifdef QLORA_DEBUG
    qlora::bounds_selftest_kernel<<<1, 1>>>(4, 4, nullptr);
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
#else
    return QLORA_ERR_UNSUPPORTED;
#endif
}

extern "C" int qlora_debug_bounds(char *unit, size_t unit_len)
{
#ifdef QLORA_DEBUG
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    qlora::BoundsRegistry &r = qlora::bounds_registry();
    std::lock_guard<std::mutex> lock(r.mu);
    int first = 0;
    for (auto &e : r.readers) {
        const int line = e.first();
        if (line != 0 && first == 0) {
            first = line;
            if (unit && unit_len) {
                const char *base = strrchr(e.second, '/');
                base = base ? base + 1 : e.second;
                strncpy(unit, base, unit_len - 1);
                unit[unit_len - 1] = 0;
            }
        }
    }
    return first;
#else
    if (unit && unit_len) unit[0] = 0;
    return -1;
#endif
}

// ---- kernel timing ------------------------------------------------------------------

namespace qlora {
namespace {
struct TimingState {
    std::mutex mu;
    bool enabled = false;
    std::vector<cudaEvent_t> pool;
    struct Rec {
        int kind;
        cudaEvent_t a, b;
    };
    std::vector<Rec> pending;
    double ms[QLORA_NUM_KERNELS] = {};
    int64_t launches[QLORA_NUM_KERNELS] = {};
};
TimingState &timing()
{
    static TimingState t;
    return t;
}
std::atomic<int64_t> g_launches{0};

cudaEvent_t take_event(TimingState &t)
{
    if (!t.pool.empty()) {
        cudaEvent_t e = t.pool.back();
        t.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

LaunchScope::LaunchScope(int kind, cudaStream_t s) : kind_(kind), s_(s)
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
    TimingState &t = timing();
    std::lock_guard<std::mutex> lock(t.mu);
    if (!t.enabled) return;
    start_ = take_event(t);
    if (start_) cudaEventRecord(start_, s_);
}

LaunchScope::~LaunchScope()
{
    if (!start_) return;
    TimingState &t = timing();
    std::lock_guard<std::mutex> lock(t.mu);
    cudaEvent_t stop = take_event(t);
    if (!stop) {
        t.pool.push_back(start_);
        return;
    }
    cudaEventRecord(stop, s_);
    t.pending.push_back({kind_, start_, stop});
}

}  // namespace qlora

extern "C" qlora_status qlora_timing_enable(int enable)
{
    TimingState &t = timing();
    std::lock_guard<std::mutex> lock(t.mu);
    t.enabled = enable != 0;
    return QLORA_OK;
}

extern "C" qlora_status qlora_timing_reset(void)
{
    TimingState &t = timing();
    std::lock_guard<std::mutex> lock(t.mu);
    for (auto &r : t.pending) {
        cudaEventSynchronize(r.b);
        t.pool.push_back(r.a);
        t.pool.push_back(r.b);
    }
    t.pending.clear();
    for (int i = 0; i < QLORA_NUM_KERNELS; i++) {
        t.ms[i] = 0.0;
        t.launches[i] = 0;
    }
    return QLORA_OK;
}

extern "C" qlora_status qlora_timing_read(double ms[QLORA_NUM_KERNELS], int64_t launches[QLORA_NUM_KERNELS])
{
    if (!ms || !launches) return QLORA_ERR_INVALID_ARG;
    TimingState &t = timing();
    std::lock_guard<std::mutex> lock(t.mu);
    qlora_status st = QLORA_OK;
    for (auto &r : t.pending) {
        float v = 0.0f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&v, r.a, r.b) != cudaSuccess)
            st = QLORA_ERR_CUDA;
        t.ms[r.kind] += v;
        t.launches[r.kind] += 1;
        t.pool.push_back(r.a);
        t.pool.push_back(r.b);
    }
    t.pending.clear();
    for (int i = 0; i < QLORA_NUM_KERNELS; i++) {
        ms[i] = t.ms[i];
        launches[i] = t.launches[i];
    }
    return st;
}

extern "C" int64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }
