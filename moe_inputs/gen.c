/*
 * Seeded synthetic inputs for the sparse MoE feed-forward layer.
 *
 * This file holds no arithmetic of the layer itself: it only fills arrays with
 * pseudo-random normal samples.  Both the fp64 CPU oracle and the CUDA path read
 * the arrays it writes, so the two sides see byte-identical inputs.
 *
 * Generator (counter based, so the value of element i does not depend on how
 * the work is split across threads):
 *   - SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the i-th output (i = 0, 1, ...) of a stream
 *     started at state s is mix64(s + (i + 1) * 0x9E3779B97F4A7C15).
 *   - The stream of tensor `tensor_id` under seed `seed` starts at
 *     s = mix64(seed * 256 + tensor_id).
 *   - A uniform in (0, 1) is u = ((r >> 11) + 0.5) * 2^-53.
 *   - Box-Muller (Box and Muller 1958): element pair p uses u1 = U(2p) and
 *     u2 = U(2p + 1); element 2p gets sqrt(-2 ln u1) cos(2 pi u2), element
 *     2p + 1 gets sqrt(-2 ln u1) sin(2 pi u2).
 *   - The sample is scaled by sigma in double, rounded to fp32 (round to
 *     nearest even), and for bf16 storage rounded again to bf16 (round to
 *     nearest even).  The stored bits are the input; nobody re-derives them.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static const uint64_t GAMMA = 0x9E3779B97F4A7C15ULL;

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline double unit_open(uint64_t r) {
    return ((double)(r >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {           /* inf / nan: keep, quiet nan */
        uint16_t h = (uint16_t)(u >> 16);
        if (u & 0x007fffffu) h |= 0x0040u;
        return h;
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* value of element i of the stream as a double, before scaling */
static inline double normal_at(uint64_t s, uint64_t i) {
    uint64_t p = i >> 1;
    double u1 = unit_open(mix64(s + (2 * p + 1) * GAMMA));
    double u2 = unit_open(mix64(s + (2 * p + 2) * GAMMA));
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint64_t stream_start(uint64_t seed, uint64_t tensor_id) {
    return mix64(seed * 256u + tensor_id);
}

/* fp32 fill: out[i] = (float)(sigma * z_i), i in [0, n) */
void moe_gen_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id, double sigma) {
    uint64_t s = stream_start(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(sigma * normal_at(s, (uint64_t)i));
}

/* bf16 fill (bit patterns): out[i] = bf16(float(sigma * z_i)) */
void moe_gen_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id, double sigma) {
    uint64_t s = stream_start(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne((float)(sigma * normal_at(s, (uint64_t)i)));
}

/* raw SplitMix64 outputs of a stream, for the generator's own tests */
void moe_gen_splitmix64(uint64_t* out, int64_t n, uint64_t state) {
    for (int64_t i = 0; i < n; ++i) out[i] = mix64(state + (uint64_t)(i + 1) * GAMMA);
}

/* bf16 rounding of fp32 values, exposed for the generator's own tests */
void moe_gen_f32_to_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

int moe_gen_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
