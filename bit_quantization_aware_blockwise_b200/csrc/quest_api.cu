// Host side of the C ABI declared in include/quest.h: argument validation,
// the alpha_b table, per-call constants and kernel dispatch. Nothing here
// allocates device memory or synchronises (except quest_device_status).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "quest.h"
#include "quest_debug.h"
#include "quest_device.cuh"
#include "quest_internal.h"

namespace quest {
namespace {

thread_local std::string g_last_error;

quest_status fail(quest_status s, const std::string& msg) {
    g_last_error = msg;
    return s;
}

quest_status cuda_fail(cudaError_t e, const char* where) {
    g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
    return QUEST_ECUDA;
}

// Fault armed by quest_debug_inject_fault for this host thread (QUEST_FAULT_NONE
// normally). take_fault consumes it when it is the one asked for.
thread_local int g_fault = QUEST_FAULT_NONE;

bool take_fault(quest_fault f) {
    if (g_fault != (int)f) return false;
    g_fault = QUEST_FAULT_NONE;
    return true;
}

quest_status injected_launch_failure(const char* where) {
    g_last_error = std::string(where) + " launch: injected launch failure (quest_debug_inject_fault); nothing launched";
    return QUEST_ECUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_had(int hb) { return hb == 16 || hb == 32 || hb == 64 || hb == 128 || hb == 256; }

// Longest row the one-RMS-per-row kernel keeps in registers: 2 passes of
// 8 warps x (32 / lanes per block) blocks.
int64_t row_mode_max_cols(int hb) { return hb == 16 ? 8192 : 16384; }

// ---------------------------------------------------------------------------
// alpha_b. The MSE of the 2^b-level midrise grid of step D on X ~ N(0,1) is
//   MSE(D) = 2 sum_{i=0}^{L-1} E[(X - (i+1/2) D)^2 ; X in cell_i],  L = 2^(b-1),
// cell_i = [iD, (i+1)D) (the last one open). Its thresholds sit midway
// between levels, so the boundary terms of d/dD cancel and
//   dMSE/dD = -4 sum_i (i+1/2) E[(X - (i+1/2) D) ; cell_i]
// The optimum is the root of  g(D) = sum_i (i+1/2)(phi(a_i) - phi(b_i))
//                                    - D sum_i (i+1/2)^2 P(cell_i),
// positive below the optimum and negative above it; it is found by bisection.
// ---------------------------------------------------------------------------
double std_normal_pdf(double x) { return isinf(x) ? 0.0 : exp(-0.5 * x * x) * 0.3989422804014327; }

double cell_prob(double a, double b) {
    const double ub = isinf(b) ? 0.0 : erfc(b * 0.7071067811865476);
    return 0.5 * (erfc(a * 0.7071067811865476) - ub);
}

double stationarity_residual(int bits, double d) {
    const int L = 1 << (bits - 1);
    double first = 0.0, second = 0.0;
    for (int i = 0; i < L; ++i) {
        const double a = i * d, b = (i == L - 1) ? INFINITY : (i + 1) * d, c = i + 0.5;
        first += c * (std_normal_pdf(a) - std_normal_pdf(b));
        second += c * c * cell_prob(a, b);
    }
    return first - d * second;
}

double optimal_step(int bits) {
    double lo = 1e-3, hi = 4.0;
    for (int it = 0; it < 200; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (stationarity_residual(bits, mid) > 0.0)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

double g_alpha[9];
std::once_flag g_alpha_once;

void init_alpha() {
    g_alpha[0] = NAN;
    for (int b = 1; b <= 8; ++b) g_alpha[b] = ldexp(optimal_step(b), b - 1);
}

// s* of the FP4 grid: the non-negative E2M1 values v_k with round-to-nearest
// cells [s (v_(k-1) + v_k) / 2, s (v_k + v_(k+1)) / 2) (the first from 0, the last
// open). The midpoint thresholds cancel the boundary terms of dMSE/ds again, so
// the optimum is the root of  g(s) = sum_k v_k (phi(a_k) - phi(b_k)) - s sum_k v_k^2 P(cell_k),
// positive below it; found by bisection.
constexpr double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double fp4_stationarity_residual(double s) {
    double first = 0.0, second = 0.0;
    for (int k = 0; k < 8; ++k) {
        const double a = k == 0 ? 0.0 : 0.5 * (kE2M1[k - 1] + kE2M1[k]) * s;
        const double b = k == 7 ? INFINITY : 0.5 * (kE2M1[k] + kE2M1[k + 1]) * s;
        first += kE2M1[k] * (std_normal_pdf(a) - std_normal_pdf(b));
        second += kE2M1[k] * kE2M1[k] * cell_prob(a, b);
    }
    return first - s * second;
}

double g_alpha_fp4 = NAN;
std::once_flag g_alpha_fp4_once;

void init_alpha_fp4() {
    double lo = 1e-2, hi = 2.0;
    for (int it = 0; it < 200; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (fp4_stationarity_residual(mid) > 0.0)
            lo = mid;
        else
            hi = mid;
    }
    g_alpha_fp4 = 0.5 * (lo + hi);
}

// alpha_b of the 2:4-sparse format: the step that minimises the MSE of the values
// that survive 2:4 pruning of an N(0,1) input. A survivor's magnitude has density
// (6F^2 - 4F^3) f (F the half-normal CDF, f its density; the mean of the 3rd and 4th
// order statistics of four samples), so a cell [a, b) holds mass G(b) - G(a) with
// G = 2F^3 - F^4; its first moment has no closed form and is taken by 64-point
// Gauss-Legendre quadrature (the last cell cut 12 beyond its start, where the
// density is below 1e-30). As for the dense grid the thresholds sit midway between
// levels, so the optimum is the root of
//   g(D) = sum_i (i+1/2) (M1_i - (i+1/2) D M0_i),
// positive below it; found by bisection.
constexpr int kGL = 64;
double g_gl_x[kGL], g_gl_w[kGL];
std::once_flag g_gl_once;

void init_gauss_legendre() {
    // nodes: roots of P_n by Newton's method from the Chebyshev guesses; weights
    // 2 / ((1 - x^2) P_n'(x)^2)
    for (int i = 0; i < kGL; ++i) {
        double x = cos(M_PI * (i + 0.75) / (kGL + 0.5)), dp = 1.0;
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = x;
            for (int n = 2; n <= kGL; ++n) {
                const double pn = ((2.0 * n - 1.0) * x * p1 - (n - 1.0) * p0) / n;
                p0 = p1;
                p1 = pn;
            }
            dp = kGL * (x * p1 - p0) / (x * x - 1.0);
            const double dx = p1 / dp;
            x -= dx;
            if (fabs(dx) < 1e-16) break;
        }
        g_gl_x[i] = x;
        g_gl_w[i] = 2.0 / ((1.0 - x * x) * dp * dp);
    }
}

double halfnormal_cdf(double a) { return erf(a * 0.7071067811865476); }
double kept_mass_antiderivative(double a) {
    if (isinf(a)) return 1.0;
    const double F = halfnormal_cdf(a);
    return 2.0 * F * F * F - F * F * F * F;
}
double kept_first_moment(double a, double b) {
    const double h = 0.5 * (b - a), m = 0.5 * (a + b);
    double acc = 0.0;
    for (int i = 0; i < kGL; ++i) {
        const double x = m + h * g_gl_x[i], F = halfnormal_cdf(x);
        acc += g_gl_w[i] * x * (6.0 * F * F - 4.0 * F * F * F) * 2.0 * std_normal_pdf(x);
    }
    return acc * h;
}

double sparse_stationarity_residual(int bits, double d) {
    const int L = 1 << (bits - 1);
    double g = 0.0;
    for (int i = 0; i < L; ++i) {
        const double a = i * d, b = (i == L - 1) ? a + 12.0 : (i + 1) * d, c = i + 0.5;
        const double m0 = kept_mass_antiderivative(i == L - 1 ? INFINITY : b) - kept_mass_antiderivative(a);
        g += c * (kept_first_moment(a, b) - c * d * m0);
    }
    return g;
}

double g_alpha_sparse[9];
std::once_flag g_alpha_sparse_once;

void init_alpha_sparse() {
    std::call_once(g_gl_once, init_gauss_legendre);
    g_alpha_sparse[0] = NAN;
    for (int b = 1; b <= 8; ++b) {
        double lo = 1e-3, hi = 6.0;
        for (int it = 0; it < 200; ++it) {
            const double mid = 0.5 * (lo + hi);
            if (mid <= lo || mid >= hi) break;
            if (sparse_stationarity_residual(b, mid) > 0.0)
                lo = mid;
            else
                hi = mid;
        }
        g_alpha_sparse[b] = ldexp(0.5 * (lo + hi), b - 1);
    }
}

bool is_fp4_mode(quest_code_mode m) { return m == QUEST_CODES_FP4_PACKED || m == QUEST_CODES_FP4_OPERAND; }

int container_bits_of(int bits) {
    static const int t[9] = {0, 1, 2, 4, 4, 8, 8, 8, 8};
    return (bits >= 1 && bits <= 8) ? t[bits] : 0;
}

int code_bits(int bits, quest_code_mode mode) {
    if (mode == QUEST_CODES_FP4_PACKED) return 4;
    return mode == QUEST_CODES_PACKED ? container_bits_of(bits) : 8;
}

// Constants of the modular code packing (see quantize_fwd.cu): a packed word is
// (sum_i bits(s_i) * mult * 2^(cb*i) + add) ^ xr, where bits(s_i) = kMagicBits
// plus the code, so that every field holds the code plus a bias in [0, 2^cb).
//
// Half-slab kernels: codes biased as q_b = q + 2^(b-1) in [0, 2^b - 1];
// field = q_b + 2^(cb-1) - 2^(b-1), or 2 q_b + 129 - 2^b for the operand form.
void pack_constants_biased(int cb, int bits, quest_code_mode mode, uint32_t* mult, uint32_t* add,
                           uint32_t* xr) {
    // the half-slab kernels pack full 32-bit words: 32, 16, 8 or 4 fields
    uint32_t rep;
    switch (cb) {
        case 1: rep = 0xFFFFFFFFu; *xr = 0xFFFFFFFFu; break;
        case 2: rep = 0x55555555u; *xr = 0xAAAAAAAAu; break;
        case 4: rep = 0x11111111u; *xr = 0x88888888u; break;
        default: rep = 0x01010101u; *xr = 0x80808080u; break;
    }
    const uint32_t half_cb = 1u << (cb - 1), half_b = 1u << (bits - 1);
    if (mode == QUEST_CODES_GEMM_OPERAND) {
        *mult = 2;
        *add = ((129u - (1u << bits)) - 2u * kMagicBits) * rep;
    } else {
        *mult = 1;
        *add = ((half_cb - half_b) - kMagicBits) * rep;
    }
}

// Direct kernels: 8 fields per word for cb < 8 (4 for cb = 8), codes q; field =
// q + 2^(cb-1), or 2 q + 1 + 128 for the operand form.
void pack_constants(int cb, quest_code_mode mode, uint32_t* mult, uint32_t* add, uint32_t* xr) {
    uint32_t bias, rep, m = 1;
    switch (cb) {
        case 1: bias = 1; rep = 0xFFu; *xr = 0xFFu; break;
        case 2: bias = 2; rep = 0x5555u; *xr = 0xAAAAu; break;
        case 4: bias = 8; rep = 0x11111111u; *xr = 0x88888888u; break;
        default: bias = 128; rep = 0x01010101u; *xr = 0x80808080u; break;
    }
    uint32_t base = bias - kMagicBits;                 // mod 2^32
    if (mode == QUEST_CODES_GEMM_OPERAND) {            // field = 2 q + 1 + 128
        m = 2;
        base = (bias + 1u) - 2u * kMagicBits;
    }
    *mult = m;
    *add = base * rep;
}

std::mutex g_occ_mutex;
std::map<std::pair<const void*, int>, int> g_occ;
std::map<int, int> g_sms;

}  // namespace

int sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_occ_mutex);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
    g_sms[dev] = n;
    return n;
}

int max_ctas_per_sm(const void* func, int threads, size_t smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_occ_mutex);
    auto key = std::make_pair(func, dev);
    auto it = g_occ.find(key);
    if (it != g_occ.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess || n <= 0)
        n = 1;
    g_occ[key] = n;
    return n;
}

}  // namespace quest

using namespace quest;

// Validates the arguments of one quantizer call and fills the kernel arguments
// (QuEST forward quantizer; see quest_quantize_fwd in quest.h). `a.rows` == 0 means
// there is nothing to launch.
static quest_status prepare_quantize(const void* x, quest_dtype x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                              int bits, int had_block, int64_t rms_group, float trust,
                              quest_code_mode code_mode, void* codes, float* scales,
                              quest_mask_mode mask_mode, void* mask, void* dequant, quest_dtype dequant_dtype,
                              QuantArgs& a, bool& row_mode, int& cb, double alpha_override = 0.0) {
    a = QuantArgs{};
    if (x_dtype != QUEST_BF16 && x_dtype != QUEST_FP32) return fail(QUEST_EINVAL, "x_dtype must be QUEST_BF16 or QUEST_FP32");
    if (rows < 0) return fail(QUEST_EINVAL, "rows must be >= 0");
    if (bits < 1 || bits > 8) return fail(QUEST_EINVAL, "bits must be in 1..8");
    if (!valid_had(had_block)) return fail(QUEST_EINVAL, "had_block must be 16, 32, 64, 128 or 256");
    if (cols <= 0 || cols % had_block != 0) return fail(QUEST_EINVAL, "cols must be a positive multiple of had_block");
    if (ld_x < cols) return fail(QUEST_EINVAL, "ld_x must be >= cols");
    if (rms_group != had_block && rms_group != cols)
        return fail(QUEST_EINVAL, "rms_group must equal had_block or cols");
    row_mode = rms_group != had_block;
    if (row_mode && cols > row_mode_max_cols(had_block))
        return fail(QUEST_EUNSUPPORTED, "rms_group == cols supports at most 16384 columns (8192 for had_block 16)");
    if (!(trust > 0.0f) || isinf(trust)) return fail(QUEST_EINVAL, "trust must be finite and > 0");
    if (code_mode != QUEST_CODES_PACKED && code_mode != QUEST_CODES_INT8 && code_mode != QUEST_CODES_GEMM_OPERAND &&
        code_mode != QUEST_CODES_GEMM_OPERAND_E4M3 && !is_fp4_mode(code_mode))
        return fail(QUEST_EINVAL, "invalid code_mode");
    const bool fp4 = is_fp4_mode(code_mode);
    if (fp4 && bits != 4) return fail(QUEST_EINVAL, "the FP4 (E2M1) grid needs bits == 4");
    if (code_mode == QUEST_CODES_GEMM_OPERAND && bits > 7)
        return fail(QUEST_EINVAL, "the GEMM operand form c = 2q+1 needs bits <= 7 to fit int8");
    if (code_mode == QUEST_CODES_GEMM_OPERAND_E4M3 && bits > 4)
        return fail(QUEST_EINVAL, "the E4M3 operand form holds c = 2q+1 exactly only for bits <= 4");
    if (mask && mask_mode != QUEST_MASK_BITS && mask_mode != QUEST_MASK_BYTES)
        return fail(QUEST_EINVAL, "invalid mask_mode");
    if (dequant && dequant_dtype != QUEST_BF16 && dequant_dtype != QUEST_FP32)
        return fail(QUEST_EINVAL, "invalid dequant_dtype");
    const int esize = x_dtype == QUEST_BF16 ? 2 : 4;
    cb = code_bits(bits, code_mode);
    if (rows > 0) {
        if (!x || !codes || !scales) return fail(QUEST_EINVAL, "x, codes and scales must be non-NULL");
        if (!aligned(x, 16) || (ld_x * esize) % 16 != 0)
            return fail(QUEST_EINVAL, "x must be 16-byte aligned with a row pitch that is a multiple of 16 bytes");
        if (!aligned(codes, cb == 8 ? 8 : (cb == 4 ? 4 : (cb == 2 ? 2 : 1))))
            return fail(QUEST_EINVAL, "codes is not aligned to its store width (8 bytes for int8 forms)");
        if (!aligned(scales, 4)) return fail(QUEST_EINVAL, "scales must be 4-byte aligned");
        if (mask && mask_mode == QUEST_MASK_BYTES && !aligned(mask, 8))
            return fail(QUEST_EINVAL, "a byte mask must be 8-byte aligned");
        if (dequant && !aligned(dequant, 16)) return fail(QUEST_EINVAL, "dequant must be 16-byte aligned");
    }
    if (rows == 0) return QUEST_OK;

    const double alpha = alpha_override > 0.0 ? alpha_override : quest_alpha(bits);
    const int lo = -(1 << (bits - 1)), hi = (1 << (bits - 1)) - 1;
    // the FP4 grid: Delta = s* r, mask edge 6 + T for T >= 1 (the last grid
    // interval [4, 6] is 2 wide, so T of its halves reach 6 + T)
    const double cd_grid = fp4 ? quest_alpha_fp4() : alpha / ldexp(1.0, bits - 1);
    const double edge_grid = fp4 ? 6.0 + (double)trust : ldexp(1.0, bits - 1) + 0.5 * ((double)trust - 1.0);
    a.x = static_cast<const char*>(x);
    a.ld_x_bytes = ld_x * esize;
    a.rows = rows;
    a.cols = cols;
    a.dense = ld_x == cols;
    a.codes = static_cast<uint8_t*>(codes);
    a.codes_row_bytes = cols * cb / 8;
    a.scales = scales;
    a.mask = static_cast<uint8_t*>(mask);
    a.mask_row_bytes = mask_mode == QUEST_MASK_BITS ? cols / 8 : cols;
    a.deq = static_cast<uint8_t*>(dequant);
    a.deq_row_bytes = cols * (dequant_dtype == QUEST_BF16 ? 2 : 4);
    QuantConsts& c = a.c;
    c.c_delta = (float)cd_grid;
    c.inv_count = (float)(1.0 / ((double)had_block * (double)rms_group));
    c.sqrt_hb = (float)sqrt((double)had_block);
    c.edge = (float)edge_grid;
    c.half_trust = 0.5f * trust;
    c.s_lo = kMagic + (float)lo;
    c.s_hi = kMagic + (float)hi;
    pack_constants(cb, fp4 ? QUEST_CODES_INT8 : code_mode, &c.pack_mult, &c.pack_add, &c.pack_xor);
    c.inv_levels = (float)ldexp(1.0, -bits);
    c.half_levels = (float)ldexp(1.0, bits - 1);
    {
        const double cd = cd_grid, ic = 1.0 / ((double)had_block * (double)rms_group);
        const double shb = sqrt((double)had_block);
        const double edge = edge_grid;
        c.delta_k = (float)(cd * sqrt(ic));
        c.inv_k = (float)(1.0 / (shb * cd * sqrt(ic)));
        c.a_k = (float)(ldexp(1.0, -bits) / (shb * cd * sqrt(ic)));
        c.thr2_k = (float)(edge * edge * shb * shb * cd * cd * ic);
    }
    c.sat_k = (float)(ldexp(1.0, bits) * (1.0 - ldexp(1.0, -23)));
    c.s_mid = kMagic + (float)ldexp(1.0, bits - 1);
    c.s_top = kMagic + (float)(ldexp(1.0, bits) - 1.0);
    c.cell_center = (float)(0.5 - ldexp(1.0, bits - 1));
    pack_constants_biased(cb, bits, code_mode == QUEST_CODES_GEMM_OPERAND_E4M3 ? QUEST_CODES_GEMM_OPERAND
                                    : fp4 ? QUEST_CODES_INT8 : code_mode,
                          &c.pack2_mult, &c.pack2_add, &c.pack2_xor);
    c.code_fp8 = code_mode == QUEST_CODES_GEMM_OPERAND_E4M3;
    c.grid_fp4 = code_mode == QUEST_CODES_FP4_PACKED ? 1 : (code_mode == QUEST_CODES_FP4_OPERAND ? 2 : 0);
    {   // an 8-field word (one chunk of 8 elements) for cb <= 4
        const uint32_t rep8 = cb == 1 ? 0xFFu : (cb == 2 ? 0x5555u : 0x11111111u);
        const uint32_t x8 = cb == 1 ? 0xFFu : (cb == 2 ? 0xAAAAu : 0x88888888u);
        const uint32_t off = (1u << (cb - 1)) - (1u << (bits - 1));
        c.pack8_add = (off - kMagicBits) * rep8;
        c.pack8_xor = x8;
    }
    c.trust_ge1 = trust >= 1.0f;
    c.mask_mode = mask ? (int)mask_mode : -1;
    c.deq_mode = dequant ? (int)dequant_dtype : -1;

    return QUEST_OK;
}

extern "C" {

int quest_version(void) { return 10000; }

double quest_alpha(int bits) {
    if (bits < 1 || bits > 8) return NAN;
    std::call_once(g_alpha_once, init_alpha);
    return g_alpha[bits];
}

double quest_alpha_sparse24(int bits) {
    if (bits < 1 || bits > 8) return NAN;
    std::call_once(g_alpha_sparse_once, init_alpha_sparse);
    return g_alpha_sparse[bits];
}

quest_status quest_quantize_sparse24(const void* x, int64_t rows, int64_t cols, int bits, int had_block,
                                     int64_t rms_group, float trust, void* codes, void* meta, float* scales,
                                     void* mask, void* dequant, void* stream) {
    g_last_error.clear();
    if (bits < 1 || bits > 7) return fail(QUEST_EINVAL, "bits must be in 1..7 (c = 2q+1 in int8)");
    if (had_block != 128) {
        if (!valid_had(had_block)) return fail(QUEST_EINVAL, "had_block must be 16, 32, 64, 128 or 256");
        return fail(QUEST_EUNSUPPORTED, "quest_quantize_sparse24: had_block must be 128");
    }
    if (rows < 0) return fail(QUEST_EINVAL, "rows must be >= 0");
    if (cols <= 0 || cols % 128 != 0) return fail(QUEST_EINVAL, "cols must be a positive multiple of 128");
    if (rms_group != 128 && rms_group != cols) return fail(QUEST_EINVAL, "rms_group must equal had_block or cols");
    const bool row_mode = rms_group != 128;
    const int64_t spr = cols / 128;
    if (row_mode && !(spr == 1 || spr == 2 || spr == 4 || spr == 8 || spr == 16))
        return fail(QUEST_EUNSUPPORTED, "quest_quantize_sparse24: one RMS per row needs cols in 128, 256, 512, 1024, 2048");
    if (rows > 0) {
        if (!x || !codes || !meta || !scales) return fail(QUEST_EINVAL, "x, codes, meta and scales must be non-NULL");
        if (!aligned(x, 16)) return fail(QUEST_EINVAL, "x must be 16-byte aligned");
        if (!aligned(codes, 8) || !aligned(meta, 4) || !aligned(scales, 4) || (mask && !aligned(mask, 4)))
            return fail(QUEST_EINVAL, "codes must be 8-byte aligned, meta, scales and mask 4-byte aligned");
        if (dequant && !aligned(dequant, 16)) return fail(QUEST_EINVAL, "dequant must be 16-byte aligned");
    }
    SparseArgs sa;
    bool rm = false;
    int cb = 0;
    const quest_status st = prepare_quantize(x, QUEST_BF16, rows, cols, cols, bits, 128, rms_group, trust,
                                             QUEST_CODES_GEMM_OPERAND, codes, scales, QUEST_MASK_BITS, mask, dequant,
                                             QUEST_BF16, sa.q, rm, cb, quest_alpha_sparse24(bits));
    if (st != QUEST_OK || sa.q.rows == 0) return st;
    sa.q.codes_row_bytes = cols / 2;
    sa.meta = static_cast<uint8_t*>(meta);
    sa.meta_row_bytes = cols / 8;
    sa.bits = bits;
    {
        const double edge = ldexp(1.0, bits - 1) + 0.5 * ((double)trust - 1.0), half_t = 0.5 * (double)trust;
        sa.prune_ratio = (float)((half_t * half_t) / (edge * edge));
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_quantize_sparse24");
    cudaError_t e = launch_quantize_sparse24(sa, row_mode, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quest_quantize_sparse24 launch");
    return QUEST_OK;
}

double quest_alpha_fp4(void) {
    std::call_once(g_alpha_fp4_once, init_alpha_fp4);
    return g_alpha_fp4;
}

int quest_container_bits(int bits) { return container_bits_of(bits); }

size_t quest_codes_bytes(int64_t rows, int64_t cols, int bits, quest_code_mode mode) {
    if (rows < 0 || cols <= 0 || bits < 1 || bits > 8) return 0;
    if (mode != QUEST_CODES_PACKED && mode != QUEST_CODES_INT8 && mode != QUEST_CODES_GEMM_OPERAND &&
        mode != QUEST_CODES_GEMM_OPERAND_E4M3 && !is_fp4_mode(mode))
        return 0;
    if (is_fp4_mode(mode) && bits != 4) return 0;
    const int cb = code_bits(bits, mode);
    if ((cols * cb) % 8 != 0) return 0;
    return (size_t)(rows * (cols * cb / 8));
}

size_t quest_mask_bytes(int64_t rows, int64_t cols, quest_mask_mode mode) {
    if (rows < 0 || cols <= 0) return 0;
    if (mode == QUEST_MASK_BITS) return cols % 8 ? 0 : (size_t)(rows * (cols / 8));
    if (mode == QUEST_MASK_BYTES) return (size_t)(rows * cols);
    return 0;
}

const char* quest_status_string(quest_status s) {
    switch (s) {
        case QUEST_OK: return "ok";
        case QUEST_EINVAL: return "invalid argument";
        case QUEST_EUNSUPPORTED: return "unsupported";
        case QUEST_ECUDA: return "CUDA error";
        case QUEST_ETIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char* quest_last_error_message(void) { return g_last_error.c_str(); }

quest_status quest_quantize_fwd(const void* x, quest_dtype x_dtype, int64_t rows, int64_t cols,
                                int64_t ld_x, int bits, int had_block, int64_t rms_group,
                                float trust, quest_code_mode code_mode, void* codes,
                                float* scales, quest_mask_mode mask_mode, void* mask,
                                void* dequant, quest_dtype dequant_dtype, void* stream) {
    g_last_error.clear();
    QuantArgs a;
    bool row_mode = false;
    int cb = 0;
    const quest_status st = prepare_quantize(x, x_dtype, rows, cols, ld_x, bits, had_block, rms_group, trust,
                                             code_mode, codes, scales, mask_mode, mask, dequant, dequant_dtype,
                                             a, row_mode, cb);
    if (st != QUEST_OK || a.rows == 0) return st;
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_quantize_fwd");
    cudaError_t e = launch_quantize(a, x_dtype, had_block, cb, bits, row_mode, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported)
        return fail(QUEST_EUNSUPPORTED, "the E4M3 operand form and the FP4 grid need rows of whole 128-value slabs, "
                                        "aligned codes and at most 16 slabs per row in row-RMS mode");
    if (e != cudaSuccess) return cuda_fail(e, "quest_quantize_fwd launch");
    return QUEST_OK;
}

quest_status quest_quantize_operands(const void* x, int64_t M, const void* w, int64_t N, int64_t K,
                                     quest_dtype dtype, int bits, int had_block, quest_code_mode code_mode,
                                     void* x_codes, float* x_scales, void* w_codes, float* w_scales,
                                     void* stream) {
    g_last_error.clear();
    QuantArgs ax, aw;
    bool rx = false, rw = false;
    int cb = 0;
    quest_status st = prepare_quantize(x, dtype, M, K, K, bits, had_block, K, 1.0f, code_mode, x_codes, x_scales,
                                       QUEST_MASK_BITS, nullptr, nullptr, QUEST_BF16, ax, rx, cb);
    if (st != QUEST_OK) return st;
    st = prepare_quantize(w, dtype, N, K, K, bits, had_block, K, 1.0f, code_mode, w_codes, w_scales,
                          QUEST_MASK_BITS, nullptr, nullptr, QUEST_BF16, aw, rw, cb);
    if (st != QUEST_OK) return st;
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_quantize_operands");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (ax.rows > 0 && aw.rows > 0 && rx && tc_path_ok(ax, dtype, had_block, cb, true) &&
        tc_path_ok(aw, dtype, had_block, cb, true)) {
        // one launch: w's rows follow x's in the row-RMS kernel
        QuantArgs a = ax;
        a.x2 = aw.x;
        a.codes2 = aw.codes;
        a.scales2 = aw.scales;
        a.rows2 = aw.rows;
        e = launch_quantize_tc(a, had_block, cb, bits, true, s);
    } else {
        if (ax.rows > 0) e = launch_quantize(ax, dtype, had_block, cb, bits, rx, s);
        if (e == cudaSuccess && aw.rows > 0) e = launch_quantize(aw, dtype, had_block, cb, bits, rw, s);
    }
    if (e == cudaErrorNotSupported)
        return fail(QUEST_EUNSUPPORTED, "the E4M3 operand form and the FP4 grid need rows of whole 128-value slabs, "
                                        "aligned codes and at most 16 slabs per row in row-RMS mode");
    if (e != cudaSuccess) return cuda_fail(e, "quest_quantize_operands launch");
    return QUEST_OK;
}

quest_status quest_trust_bwd(const void* grad_out, const void* mask, quest_mask_mode mask_mode,
                             int64_t rows, int64_t cols, int had_block, void* grad_in,
                             void* stream) {
    g_last_error.clear();
    if (rows < 0) return fail(QUEST_EINVAL, "rows must be >= 0");
    if (!valid_had(had_block)) return fail(QUEST_EINVAL, "had_block must be 16, 32, 64, 128 or 256");
    if (cols <= 0 || cols % had_block != 0) return fail(QUEST_EINVAL, "cols must be a positive multiple of had_block");
    if (mask_mode != QUEST_MASK_BITS && mask_mode != QUEST_MASK_BYTES) return fail(QUEST_EINVAL, "invalid mask_mode");
    if (rows > 0) {
        if (!grad_out || !mask || !grad_in) return fail(QUEST_EINVAL, "grad_out, mask and grad_in must be non-NULL");
        if (!aligned(grad_out, 16) || !aligned(grad_in, 16))
            return fail(QUEST_EINVAL, "grad_out and grad_in must be 16-byte aligned");
        if (mask_mode == QUEST_MASK_BYTES && !aligned(mask, 8))
            return fail(QUEST_EINVAL, "a byte mask must be 8-byte aligned");
        const char* go = static_cast<const char*>(grad_out);
        const char* gi = static_cast<const char*>(grad_in);
        const int64_t bytes = rows * cols * 2;
        if (gi < go + bytes && go < gi + bytes) return fail(QUEST_EINVAL, "grad_in must not overlap grad_out");
    }
    if (rows == 0) return QUEST_OK;
    TrustArgs a;
    a.g = static_cast<const uint16_t*>(grad_out);
    a.mask = static_cast<const uint8_t*>(mask);
    a.mask_mode = (int)mask_mode;
    a.rows = rows;
    a.cols = cols;
    a.out = static_cast<uint16_t*>(grad_in);
    a.inv_sqrt_hb = (float)(1.0 / sqrt((double)had_block));
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_trust_bwd");
    cudaError_t e = launch_trust_bwd(a, had_block, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quest_trust_bwd launch");
    return QUEST_OK;
}

quest_status quest_w4a4_linear(const int8_t* a_codes, const float* a_scales,
                               const int8_t* w_codes, const float* w_scales, int64_t M,
                               int64_t N, int64_t K, void* y, int32_t* acc, void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return fail(QUEST_EINVAL, "M and N must be < 2^31");
    if (K % 16 != 0) return fail(QUEST_EINVAL, "K must be a multiple of 16");
    if (K >= 131072) return fail(QUEST_EINVAL, "K must be < 131072 (int32 accumulator bound)");
    if (N % 8 != 0) return fail(QUEST_EINVAL, "N must be a multiple of 8");
    if (M > 0 && N > 0) {
        if (!y || !a_scales || !w_scales) return fail(QUEST_EINVAL, "y and the scales must be non-NULL");
        if (K > 0 && (!a_codes || !w_codes)) return fail(QUEST_EINVAL, "codes must be non-NULL");
        if (K > 0 && (!aligned(a_codes, 16) || !aligned(w_codes, 16)))
            return fail(QUEST_EINVAL, "codes must be 16-byte aligned");
        if (!aligned(y, 16)) return fail(QUEST_EINVAL, "y must be 16-byte aligned");
        if (!aligned(a_scales, 4) || !aligned(w_scales, 4) || (acc && !aligned(acc, 4)))
            return fail(QUEST_EINVAL, "scales and acc must be 4-byte aligned");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_w4a4_linear");
    const bool inject_timeout = take_fault(QUEST_FAULT_WAIT_TIMEOUT);
    cudaError_t e = launch_w4a4(a_codes, a_scales, w_codes, w_scales, M, N, K,
                                static_cast<uint16_t*>(y), acc, static_cast<cudaStream_t>(stream), inject_timeout);
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_w4a4_linear: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_w4a4_linear launch");
    return QUEST_OK;
}

quest_status quest_w4a4_linear_sparse24(const int8_t* x_codes, const float* x_scales, const int8_t* w_codes,
                                        const uint8_t* w_meta, const float* w_scales, int64_t M, int64_t N, int64_t K,
                                        void* y, int32_t* acc, void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return fail(QUEST_EINVAL, "M and N must be < 2^31");
    if (K % 128 != 0) return fail(QUEST_EINVAL, "K must be a multiple of 128");
    if (K >= 131072) return fail(QUEST_EINVAL, "K must be < 131072 (int32 accumulator bound)");
    if (N % 8 != 0) return fail(QUEST_EINVAL, "N must be a multiple of 8");
    if (M > 0 && N > 0) {
        if (!y || !x_scales || !w_scales) return fail(QUEST_EINVAL, "y and the scales must be non-NULL");
        if (K > 0 && (!x_codes || !w_codes || !w_meta)) return fail(QUEST_EINVAL, "codes and meta must be non-NULL");
        if (K > 0 && (!aligned(x_codes, 16) || !aligned(w_codes, 16) || !aligned(w_meta, 16)))
            return fail(QUEST_EINVAL, "codes and meta must be 16-byte aligned");
        if (!aligned(y, 16)) return fail(QUEST_EINVAL, "y must be 16-byte aligned");
        if (!aligned(x_scales, 4) || !aligned(w_scales, 4) || (acc && !aligned(acc, 4)))
            return fail(QUEST_EINVAL, "scales and acc must be 4-byte aligned");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_w4a4_linear_sparse24");
    cudaError_t e = launch_w4a4_sparse24(x_codes, x_scales, w_codes, w_meta, w_scales, M, N, K,
                                         static_cast<uint16_t*>(y), acc, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_w4a4_linear_sparse24: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_w4a4_linear_sparse24 launch");
    return QUEST_OK;
}

quest_status quest_fp4_linear(const uint8_t* a_codes, const float* a_scales, const uint8_t* w_codes,
                              const float* w_scales, int64_t M, int64_t N, int64_t K, void* y, float* acc,
                              void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return fail(QUEST_EINVAL, "M and N must be < 2^31");
    if (K % 32 != 0) return fail(QUEST_EINVAL, "K must be a multiple of 32");
    if (K > 16384) return fail(QUEST_EINVAL, "K must be <= 16384 (exact fp32 accumulation bound)");
    if (N % 8 != 0) return fail(QUEST_EINVAL, "N must be a multiple of 8");
    if (M > 0 && N > 0) {
        if (!y) return fail(QUEST_EINVAL, "y must be non-NULL");
        if (K > 0 && (!a_codes || !w_codes || !a_scales || !w_scales))
            return fail(QUEST_EINVAL, "codes and scales must be non-NULL");
        if (K > 0 && (!aligned(a_codes, 16) || !aligned(w_codes, 16)))
            return fail(QUEST_EINVAL, "codes must be 16-byte aligned");
        if (!aligned(y, 16)) return fail(QUEST_EINVAL, "y must be 16-byte aligned");
        if ((a_scales && !aligned(a_scales, 4)) || (w_scales && !aligned(w_scales, 4)) || (acc && !aligned(acc, 4)))
            return fail(QUEST_EINVAL, "scales and acc must be 4-byte aligned");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_fp4_linear");
    cudaError_t e = launch_fp4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K, static_cast<uint16_t*>(y), acc,
                                      static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_fp4_linear: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_fp4_linear launch");
    return QUEST_OK;
}

quest_status quest_w4a4_linear_grouped(const uint8_t* a_codes, const float* a_scales,
                                       const uint8_t* w_codes, const float* w_scales, int64_t M,
                                       int64_t N, int64_t K, int64_t group, void* y, float* y_f32,
                                       void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return fail(QUEST_EINVAL, "M and N must be < 2^31");
    if (group != 128) return fail(QUEST_EUNSUPPORTED, "quest_w4a4_linear_grouped: group must be 128");
    if (K % group != 0) return fail(QUEST_EINVAL, "K must be a multiple of the group");
    if (K >= (int64_t(1) << 24)) return fail(QUEST_EINVAL, "K must be < 2^24");
    if (N % 8 != 0) return fail(QUEST_EINVAL, "N must be a multiple of 8");
    if (M > 0 && N > 0) {
        if (!y) return fail(QUEST_EINVAL, "y must be non-NULL");
        if (K > 0 && (!a_codes || !w_codes || !a_scales || !w_scales))
            return fail(QUEST_EINVAL, "codes and scales must be non-NULL");
        if (K > 0 && (!aligned(a_codes, 16) || !aligned(w_codes, 16)))
            return fail(QUEST_EINVAL, "codes must be 16-byte aligned");
        if (!aligned(y, 16)) return fail(QUEST_EINVAL, "y must be 16-byte aligned");
        if ((a_scales && !aligned(a_scales, 4)) || (w_scales && !aligned(w_scales, 4)) ||
            (y_f32 && !aligned(y_f32, 4)))
            return fail(QUEST_EINVAL, "scales and y_f32 must be 4-byte aligned");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_w4a4_linear_grouped");
    cudaError_t e = launch_w4a4_grouped(reinterpret_cast<const int8_t*>(a_codes), a_scales,
                                        reinterpret_cast<const int8_t*>(w_codes), w_scales, M, N, K,
                                        static_cast<uint16_t*>(y), y_f32, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_w4a4_linear_grouped: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_w4a4_linear_grouped launch");
    return QUEST_OK;
}

quest_status quest_trust_bwd_linear(const void* grad_y, const void* w_hat_t, const void* mask, int64_t M,
                                    int64_t N, int64_t K, int had_block, void* grad_x, void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return fail(QUEST_EINVAL, "M, N and K must be < 2^31");
    if (!valid_had(had_block)) return fail(QUEST_EINVAL, "had_block must be 16, 32, 64, 128 or 256");
    if (had_block != 128) return fail(QUEST_EUNSUPPORTED, "quest_trust_bwd_linear: had_block must be 128");
    if (K % 128 != 0) return fail(QUEST_EINVAL, "K must be a multiple of 128");
    if (N % 8 != 0) return fail(QUEST_EINVAL, "N must be a multiple of 8 (16-byte rows)");
    if (M > 0 && K > 0) {
        if (!grad_x || !mask) return fail(QUEST_EINVAL, "mask and grad_x must be non-NULL");
        if (N > 0 && (!grad_y || !w_hat_t)) return fail(QUEST_EINVAL, "grad_y and w_hat_t must be non-NULL");
        if (!aligned(grad_x, 16) || !aligned(mask, 16) || (N > 0 && (!aligned(grad_y, 16) || !aligned(w_hat_t, 16))))
            return fail(QUEST_EINVAL, "grad_y, w_hat_t, mask and grad_x must be 16-byte aligned");
        // grad_x is written while the other three are read
        const char* gx = static_cast<const char*>(grad_x);
        const int64_t gx_bytes = M * K * 2;
        auto overlaps = [&](const void* p, int64_t bytes) {
            const char* c = static_cast<const char*>(p);
            return c != nullptr && bytes > 0 && c < gx + gx_bytes && gx < c + bytes;
        };
        if (overlaps(grad_y, M * N * 2) || overlaps(w_hat_t, K * N * 2) || overlaps(mask, M * K / 8))
            return fail(QUEST_EINVAL, "grad_x must not overlap grad_y, w_hat_t or mask");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_trust_bwd_linear");
    cudaError_t e = launch_trust_linear(static_cast<const uint16_t*>(grad_y), static_cast<const uint16_t*>(w_hat_t),
                                        static_cast<const uint8_t*>(mask), M, N, K, static_cast<uint16_t*>(grad_x),
                                        static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_trust_bwd_linear: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_trust_bwd_linear launch");
    return QUEST_OK;
}

quest_status quest_linear_bf16(const void* x_hat, const void* w_hat, int64_t M, int64_t N, int64_t K, void* y,
                               void* stream) {
    g_last_error.clear();
    if (M < 0 || N < 0 || K < 0) return fail(QUEST_EINVAL, "M, N and K must be >= 0");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return fail(QUEST_EINVAL, "M, N and K must be < 2^31");
    if (K % 8 != 0 || N % 8 != 0) return fail(QUEST_EINVAL, "K and N must be multiples of 8 (16-byte rows)");
    if (M > 0 && N > 0) {
        if (!y) return fail(QUEST_EINVAL, "y must be non-NULL");
        if (K > 0 && (!x_hat || !w_hat)) return fail(QUEST_EINVAL, "x_hat and w_hat must be non-NULL");
        if (!aligned(y, 16) || (K > 0 && (!aligned(x_hat, 16) || !aligned(w_hat, 16))))
            return fail(QUEST_EINVAL, "x_hat, w_hat and y must be 16-byte aligned");
        const char* yc = static_cast<const char*>(y);
        const int64_t y_bytes = M * N * 2;
        auto overlaps = [&](const void* p, int64_t bytes) {
            const char* c = static_cast<const char*>(p);
            return c != nullptr && bytes > 0 && c < yc + y_bytes && yc < c + bytes;
        };
        if (overlaps(x_hat, M * K * 2) || overlaps(w_hat, N * K * 2))
            return fail(QUEST_EINVAL, "y must not overlap x_hat or w_hat");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_linear_bf16");
    cudaError_t e = launch_linear_bf16(static_cast<const uint16_t*>(x_hat), static_cast<const uint16_t*>(w_hat), M,
                                       N, K, static_cast<uint16_t*>(y), static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return fail(QUEST_ECUDA, "quest_linear_bf16: tensor map encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "quest_linear_bf16 launch");
    return QUEST_OK;
}

quest_status quest_transpose_bf16(const void* src, int64_t rows, int64_t cols, void* dst, void* stream) {
    g_last_error.clear();
    if (rows < 0 || cols < 0) return fail(QUEST_EINVAL, "rows and cols must be >= 0");
    if (rows > 0 && cols > 0) {
        if (!src || !dst) return fail(QUEST_EINVAL, "src and dst must be non-NULL");
        if (!aligned(src, 2) || !aligned(dst, 2)) return fail(QUEST_EINVAL, "src and dst must be 2-byte aligned");
        const char* a = static_cast<const char*>(src);
        const char* b = static_cast<const char*>(dst);
        const int64_t bytes = rows * cols * 2;
        if (a < b + bytes && b < a + bytes) return fail(QUEST_EINVAL, "src and dst must not overlap");
    }
    if (take_fault(QUEST_FAULT_LAUNCH)) return injected_launch_failure("quest_transpose_bf16");
    cudaError_t e = launch_transpose_bf16(static_cast<const uint16_t*>(src), rows, cols, static_cast<uint16_t*>(dst),
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quest_transpose_bf16 launch");
    return QUEST_OK;
}

quest_status quest_debug_inject_fault(quest_fault fault) {
    g_last_error.clear();
    if (fault != QUEST_FAULT_NONE && fault != QUEST_FAULT_LAUNCH && fault != QUEST_FAULT_WAIT_TIMEOUT)
        return fail(QUEST_EINVAL, "unknown fault");
    g_fault = (int)fault;
    return QUEST_OK;
}

quest_status quest_device_status(void* stream) {
    g_last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    // every status word is read and cleared, so a later call starts clean
    const int vg = read_and_clear_gemm_status(s, &e);
    if (e != cudaSuccess) return cuda_fail(e, "quest_device_status");
    const int vgr = read_and_clear_grouped_status(s, &e);
    if (e != cudaSuccess) return cuda_fail(e, "quest_device_status");
    const int vtl = read_and_clear_trust_linear_status(s, &e);
    if (e != cudaSuccess) return cuda_fail(e, "quest_device_status");
    const int vf4 = read_and_clear_fp4_status(s, &e);
    if (e != cudaSuccess) return cuda_fail(e, "quest_device_status");
    const int vsp = read_and_clear_sparse_status(s, &e);
    if (e != cudaSuccess) return cuda_fail(e, "quest_device_status");
    if (vg != 0) return fail((quest_status)vg, "a bounded device-side wait in quest_w4a4_linear gave up");
    if (vgr != 0) return fail((quest_status)vgr, "a bounded device-side wait in quest_w4a4_linear_grouped gave up");
    if (vtl != 0)
        return fail((quest_status)vtl, "a bounded device-side wait in quest_trust_bwd_linear or quest_linear_bf16 gave up");
    if (vf4 != 0) return fail((quest_status)vf4, "a bounded device-side wait in quest_fp4_linear gave up");
    if (vsp != 0) return fail((quest_status)vsp, "a bounded device-side wait in quest_w4a4_linear_sparse24 gave up");
    return QUEST_OK;
}

}  // extern "C"
