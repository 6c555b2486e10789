// Host side of a HARP plan: schedule validation, strides, theta layout, the sign
// diagonal and the base mixers G_b (HARP technical summary §2.1 Core
// Architecture, §2.2 Hadamard Preconditioning).  No CUDA call is made here.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include "harp_internal.h"

namespace {

thread_local std::string g_last_error;
thread_local std::string g_last_kernel;

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kQrSeedBase = 0x4841525000000000ull;

// SplitMix64 (Steele, Lea & Flood 2014): advance by the golden gamma, then mix.
struct SplitMix64 {
    uint64_t state;
    explicit SplitMix64(uint64_t seed) : state(seed) {}
    uint64_t next() {
        state += kGamma;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
};

inline double unit53(uint64_t u) { return (double)(u >> 11) * 0x1.0p-53; }

bool is_pow2(int b) { return b > 0 && (b & (b - 1)) == 0; }

// Normalized Sylvester Hadamard: (-1)^popcount(k & l) / sqrt(b).
void sylvester(int b, double* g) {
    const double inv = 1.0 / std::sqrt((double)b);
    for (int k = 0; k < b; ++k)
        for (int l = 0; l < b; ++l)
            g[k * b + l] = (__builtin_popcount((unsigned)(k & l)) & 1) ? -inv : inv;
}

// Orthogonal fallback for non-power-of-two radices: Q of a seeded Gaussian
// matrix, with column signs chosen so that R's diagonal is non-negative.
void qr_fallback(int b, uint64_t seed, double* g) {
    double a[HARP_MAX_RADIX * HARP_MAX_RADIX];
    SplitMix64 rng(seed);
    for (int e = 0; e < b * b; ++e) {
        const double u1 = unit53(rng.next());
        const double u2 = unit53(rng.next());
        a[e] = std::sqrt(-2.0 * std::log(1.0 - u1)) * std::cos(2.0 * M_PI * u2);
    }
    // Householder QR: reflect column k below the diagonal onto e_k, accumulating Q.
    double q[HARP_MAX_RADIX * HARP_MAX_RADIX];
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) q[i * b + j] = (i == j) ? 1.0 : 0.0;
    for (int k = 0; k < b; ++k) {
        double norm2 = 0.0;
        for (int i = k; i < b; ++i) norm2 += a[i * b + k] * a[i * b + k];
        const double norm = std::sqrt(norm2);
        if (norm == 0.0) continue;
        const double alpha = (a[k * b + k] >= 0.0) ? -norm : norm;
        double v[HARP_MAX_RADIX];
        for (int i = 0; i < b; ++i) v[i] = 0.0;
        for (int i = k; i < b; ++i) v[i] = a[i * b + k];
        v[k] -= alpha;
        double vv = 0.0;
        for (int i = k; i < b; ++i) vv += v[i] * v[i];
        if (vv == 0.0) continue;
        // A <- (I - 2 v v^T / v^T v) A
        for (int j = 0; j < b; ++j) {
            double dot = 0.0;
            for (int i = k; i < b; ++i) dot += v[i] * a[i * b + j];
            const double f = 2.0 * dot / vv;
            for (int i = k; i < b; ++i) a[i * b + j] -= f * v[i];
        }
        // Q <- Q (I - 2 v v^T / v^T v)
        for (int i = 0; i < b; ++i) {
            double dot = 0.0;
            for (int j = k; j < b; ++j) dot += q[i * b + j] * v[j];
            const double f = 2.0 * dot / vv;
            for (int j = k; j < b; ++j) q[i * b + j] -= f * v[j];
        }
    }
    for (int j = 0; j < b; ++j) {
        const double sg = (a[j * b + j] < 0.0) ? -1.0 : 1.0;
        for (int i = 0; i < b; ++i) g[i * b + j] = q[i * b + j] * sg;
    }
}

harp_status validate_schedule(int64_t d, const int32_t* radices, int32_t m) {
    if (!radices) return harp_fail(HARP_ERR_INVALID_ARG, "radices is NULL");
    if (m < 1 || m > HARP_MAX_STAGES)
        return harp_fail(HARP_ERR_SCHEDULE, "stage count outside [1, 16]");
    int64_t prod = 1;
    for (int t = 0; t < m; ++t) {
        if (radices[t] < 2 || radices[t] > HARP_MAX_RADIX)
            return harp_fail(HARP_ERR_SCHEDULE, "radix outside [2, 16] at stage " + std::to_string(t));
        prod *= radices[t];
        if (prod > HARP_MAX_DIM) return harp_fail(HARP_ERR_SCHEDULE, "product of radices exceeds the maximum dimension");
    }
    if (d >= 0 && prod != d)
        return harp_fail(HARP_ERR_SCHEDULE, "product of radices (" + std::to_string(prod) +
                                                ") differs from d (" + std::to_string(d) + ")");
    return HARP_OK;
}

}  // namespace

harp_status harp_fail(harp_status s, const std::string& msg) {
    g_last_error = std::string(harp_status_string(s)) + ": " + msg;
    return s;
}

void harp_clear_error() { g_last_error.clear(); }

void harp_set_last_kernel(const char* name) { g_last_kernel = name; }

extern "C" {

const char* harp_status_string(harp_status s) {
    switch (s) {
        case HARP_OK: return "HARP_OK";
        case HARP_ERR_INVALID_ARG: return "HARP_ERR_INVALID_ARG";
        case HARP_ERR_SCHEDULE: return "HARP_ERR_SCHEDULE";
        case HARP_ERR_UNSUPPORTED: return "HARP_ERR_UNSUPPORTED";
        case HARP_ERR_NOT_MATERIALIZED: return "HARP_ERR_NOT_MATERIALIZED";
        case HARP_ERR_ALLOC: return "HARP_ERR_ALLOC";
        case HARP_ERR_CUDA: return "HARP_ERR_CUDA";
        case HARP_ERR_TIMEOUT: return "HARP_ERR_TIMEOUT";
        case HARP_ERR_WRONG_DEVICE: return "HARP_ERR_WRONG_DEVICE";
    }
    return "HARP_ERR_UNKNOWN";
}

const char* harp_last_error(void) { return g_last_error.c_str(); }

const char* harp_last_kernel(void) { return g_last_kernel.c_str(); }

int64_t harp_theta_count(const int32_t* radices, int32_t m) {
    if (validate_schedule(-1, radices, m) != HARP_OK) return -1;
    int64_t d = 1;
    for (int t = 0; t < m; ++t) d *= radices[t];
    int64_t n = 0;
    for (int t = 0; t < m; ++t) {
        const int b = radices[t];
        n += (d / b) * (b == 2 ? 1 : b * (b - 1) / 2);
    }
    return n;
}

harp_status harp_splitmix64(uint64_t seed, int64_t n, uint64_t* out) {
    if (n < 0 || (n > 0 && !out)) return harp_fail(HARP_ERR_INVALID_ARG, "bad output array");
    SplitMix64 rng(seed);
    for (int64_t i = 0; i < n; ++i) out[i] = rng.next();
    return HARP_OK;
}

harp_status harp_plan_create(harp_plan_t* out, int64_t d, const int32_t* radices, int32_t m,
                             harp_theta_kind kind, const void* theta, const float* scales,
                             uint64_t sign_seed, uint64_t qr_seed) {
    harp_clear_error();
    if (!out) return harp_fail(HARP_ERR_INVALID_ARG, "out is NULL");
    if (d < 2 || d > HARP_MAX_DIM) return harp_fail(HARP_ERR_INVALID_ARG, "d outside [2, 32768]");
    harp_status st = validate_schedule(d, radices, m);
    if (st != HARP_OK) return st;
    if (kind != HARP_THETA_F32 && kind != HARP_THETA_I8)
        return harp_fail(HARP_ERR_UNSUPPORTED, "unknown theta kind");
    if (kind == HARP_THETA_I8 && theta && !scales)
        return harp_fail(HARP_ERR_INVALID_ARG, "int8 theta needs per-stage scales");

    harp_plan_s* p = new (std::nothrow) harp_plan_s();
    if (!p) return harp_fail(HARP_ERR_ALLOC, "host allocation of the plan");
    try {
        p->desc.d = d;
        p->desc.m = m;
        p->kind = kind;
        p->sign_seed = sign_seed;
        p->qr_seed = qr_seed;
        int64_t s = 1, toff = 0, boff = 0, loff = 0;
        for (int t = 0; t < m; ++t) {
            StageDesc& sd = p->desc.st[t];
            sd.b = radices[t];
            sd.p = sd.b == 2 ? 1 : sd.b * (sd.b - 1) / 2;
            sd.s = s;
            sd.nblocks = d / sd.b;
            sd.theta_off = toff;
            sd.block_off = boff;
            p->lane_off[t] = loff;
            s *= sd.b;
            toff += sd.nblocks * sd.p;
            boff += sd.nblocks * sd.b * sd.b;
            loff += (sd.nblocks + 31) / 32 * 32 * sd.b * sd.b;
        }
        p->theta_total = toff;
        p->block_floats = boff;
        p->lane_floats = loff;

        if (kind == HARP_THETA_F32) {
            p->theta_f32.assign(toff, 0.0f);
            if (theta) std::memcpy(p->theta_f32.data(), theta, toff * sizeof(float));
            p->scales.assign(m, 1.0f);
        } else {
            p->theta_i8.assign(toff, 0);
            if (theta) std::memcpy(p->theta_i8.data(), theta, toff);
            p->scales.assign(m, 1.0f);
            if (scales) std::memcpy(p->scales.data(), scales, m * sizeof(float));
        }

        p->signs.resize(d);
        SplitMix64 rng(sign_seed);
        for (int64_t i = 0; i < d; ++i) p->signs[i] = (rng.next() >> 63) ? -1 : 1;

        for (int t = 0; t < m; ++t) {
            const int b = p->desc.st[t].b;
            if (p->mixer_index.count(b) == 0) {
                const int off = (int)p->mixers.size();
                p->mixers.resize(off + b * b);
                if (is_pow2(b))
                    sylvester(b, p->mixers.data() + off);
                else
                    qr_fallback(b, (qr_seed ? qr_seed : kQrSeedBase) + (uint64_t)b, p->mixers.data() + off);
                p->mixer_index[b] = off;
            }
            p->desc.st[t].mixer_off = p->mixer_index[b];
        }
    } catch (const std::bad_alloc&) {
        delete p;
        return harp_fail(HARP_ERR_ALLOC, "host allocation of plan arrays");
    }
    *out = p;
    return HARP_OK;
}

harp_status harp_plan_destroy(harp_plan_t plan) {
    if (!plan) return HARP_OK;
    harp_status st = harp_device_free(plan);
    delete plan;
    return st;
}

harp_status harp_plan_base_mixer(harp_plan_t plan, int32_t radix, double* out) {
    if (!plan || !out) return harp_fail(HARP_ERR_INVALID_ARG, "NULL argument");
    if (plan->composite) return harp_fail(HARP_ERR_UNSUPPORTED, "a composite has the mixers of its plans");
    auto it = plan->mixer_index.find(radix);
    if (it == plan->mixer_index.end()) return harp_fail(HARP_ERR_INVALID_ARG, "radix not in the plan");
    std::memcpy(out, plan->mixers.data() + it->second, sizeof(double) * radix * radix);
    return HARP_OK;
}

harp_status harp_plan_signs(harp_plan_t plan, int8_t* out) {
    if (!plan || !out) return harp_fail(HARP_ERR_INVALID_ARG, "NULL argument");
    if (plan->composite) return harp_fail(HARP_ERR_UNSUPPORTED, "a composite has the signs of its plans");
    std::memcpy(out, plan->signs.data(), plan->signs.size());
    return HARP_OK;
}

harp_status harp_plan_shape(harp_plan_t plan, int64_t* d, int32_t* m, int32_t* radices) {
    if (!plan) return harp_fail(HARP_ERR_INVALID_ARG, "NULL plan");
    if (d) *d = plan->desc.d;
    if (m) *m = plan->desc.m;
    if (radices)
        for (int t = 0; t < HARP_MAX_STAGES; ++t) radices[t] = t < plan->desc.m ? plan->desc.st[t].b : 0;
    return HARP_OK;
}

}  // extern "C"
