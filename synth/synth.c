/*
 * Seeded synthetic Q/K/V generator for 3D block sparse attention workloads.
 *
 * This module produces INPUTS only. It holds none of the attention method's
 * arithmetic (no chunking, pooling, scoring, selection or softmax), and it is
 * shared by the CPU oracle, the GPU tests and the benchmark so that both sides
 * read bit-identical bf16 tensors.
 *
 * What it models. The attention operator of a video DiT consumes Q, K and V
 * after the projections and QK-RMSNorm ("LongCat-Video Technical Report",
 * section "Model Architecture": RMSNorm on queries and keys; section
 * "Block Sparse Attention (BSA)": Q = X W_q, K = X W_k with layout
 * [b, n_h, T*H*W, d] in [T,H,W] memory order). Video latents are spatially and
 * temporally smooth, which is the redundancy BSA exploits (same section, "video
 * latent redundancy"). Each (batch, head, tensor) is therefore a smooth field:
 *
 *   x[t,h,w,c] = sum_{i<4} u_i[c] * sin(2*pi*(ft_i*t/T + fh_i*h/H + fw_i*w/W) + phi_i)
 *                + 0.3 * n[t,h,w,c],          n ~ N(0,1)
 *
 * with ft_i, fh_i, fw_i ~ U[0,2) cycles per axis extent (ft scaled by
 * `tfreq_mult` to emulate faster motion), phi_i ~ U[0,2*pi), u_i[c] ~ U[-1,1).
 * Q and K are then RMS-normalised per token, x / sqrt(mean_c(x^2) + 1e-6), with
 * no learned gain; V is not normalised. All arithmetic is in double, rounded to
 * float (round-to-nearest-even) and then to bf16 (round-to-nearest-even).
 *
 * Frames t < cond_frames are drawn from `cond_seed` instead of `seed` (the
 * condition frames of a video-continuation input come from a different clip).
 *
 * Random numbers. A counter-based generator: the SplitMix64 output function
 * (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014) applied to key + (counter+1)*golden-gamma. A uniform in [0,1) is
 * the top 53 bits times 2^-53. Normals use the Box-Muller transform on
 * consecutive counter pairs. Stream keys are derived from
 * (seed, tensor, batch, head, component) by chaining the same mixer, so every
 * element is addressable without generating its predecessors.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL
#define NOISE_COMPONENT 99u

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t ctr_u64(uint64_t key, uint64_t ctr) {
    return mix64(key + (ctr + 1ULL) * GOLDEN_GAMMA);
}

static inline double ctr_u01(uint64_t key, uint64_t ctr) {
    return (double)(ctr_u64(key, ctr) >> 11) * 0x1.0p-53;
}

static uint64_t stream_key(uint64_t seed, uint32_t tensor, uint32_t b, uint32_t head,
                           uint32_t comp) {
    uint64_t h = mix64(seed + GOLDEN_GAMMA);
    h = mix64(h ^ ((uint64_t)tensor + 0x100ULL));
    h = mix64(h ^ ((uint64_t)b + 0x10000ULL));
    h = mix64(h ^ ((uint64_t)head + 0x1000000ULL));
    h = mix64(h ^ ((uint64_t)comp + 0x100000000ULL));
    return h;
}

/* Standard normal number `idx` of a stream (Box-Muller on counter pair). */
static inline double ctr_normal(uint64_t key, uint64_t idx) {
    uint64_t pair = idx >> 1;
    double u1 = 1.0 - ctr_u01(key, 2 * pair); /* (0,1] so log is finite */
    double u2 = ctr_u01(key, 2 * pair + 1);
    double r = sqrt(-2.0 * log(u1));
    double a = 2.0 * M_PI * u2;
    return (idx & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

#define NCOMP 4
#define MAX_D 256

typedef struct {
    double ft, fh, fw, phi;
    double u[MAX_D];
} component_t;

static void make_components(component_t* cp, uint64_t seed, uint32_t tensor, uint32_t b,
                            uint32_t head, int d, double tfreq_mult) {
    for (int i = 0; i < NCOMP; ++i) {
        uint64_t key = stream_key(seed, tensor, b, head, (uint32_t)i);
        cp[i].ft = 2.0 * ctr_u01(key, 0) * tfreq_mult;
        cp[i].fh = 2.0 * ctr_u01(key, 1);
        cp[i].fw = 2.0 * ctr_u01(key, 2);
        cp[i].phi = 2.0 * M_PI * ctr_u01(key, 3);
        for (int c = 0; c < d; ++c) cp[i].u[c] = 2.0 * ctr_u01(key, 4 + (uint64_t)c) - 1.0;
    }
}

/*
 * Fill out[B][heads][T][H][W][d] (bf16 bit patterns) for one tensor. Batch
 * element b uses stream batch index b + b_offset and head hd stream head index
 * hd + h_offset, so disjoint slices of a large virtual problem (a range of batch
 * elements, or a range of heads of one batch element) can be generated
 * independently, e.g. one per rank.
 * tensor: 0 = Q, 1 = K, 2 = V (selects the stream; also any other id works).
 * rms_norm: 1 to RMS-normalise each token (Q, K), 0 for V.
 * Returns 0 on success, -1 on bad arguments.
 */
int synth_field_bf16_slice(uint16_t* out, int B, int b_offset, int heads, int h_offset, int T,
                           int H, int W, int d, uint64_t seed, uint32_t tensor, int rms_norm,
                           double tfreq_mult, int cond_frames, uint64_t cond_seed) {
    if (!out || B <= 0 || b_offset < 0 || heads <= 0 || h_offset < 0 || T <= 0 || H <= 0 ||
        W <= 0 || d <= 0 || d > MAX_D || (d & 1))
        return -1;
    const int64_t N = (int64_t)T * H * W;
    for (int b = 0; b < B; ++b) {
        for (int hd = 0; hd < heads; ++hd) {
            component_t comp_main[NCOMP], comp_cond[NCOMP];
            const uint32_t bs = (uint32_t)(b + b_offset);
            const uint32_t hs = (uint32_t)(hd + h_offset);
            make_components(comp_main, seed, tensor, bs, hs, d, tfreq_mult);
            make_components(comp_cond, cond_seed, tensor, bs, hs, d, tfreq_mult);
            const uint64_t nkey_main = stream_key(seed, tensor, bs, hs, NOISE_COMPONENT);
            const uint64_t nkey_cond = stream_key(cond_seed, tensor, bs, hs, NOISE_COMPONENT);
            uint16_t* base = out + ((int64_t)b * heads + hd) * N * d;
#pragma omp parallel for schedule(static)
            for (int64_t tok = 0; tok < N; ++tok) {
                const int t = (int)(tok / ((int64_t)H * W));
                const int h = (int)((tok / W) % H);
                const int w = (int)(tok % W);
                const int is_cond = t < cond_frames;
                const component_t* cp = is_cond ? comp_cond : comp_main;
                const uint64_t nkey = is_cond ? nkey_cond : nkey_main;
                double s[NCOMP];
                for (int i = 0; i < NCOMP; ++i)
                    s[i] = sin(2.0 * M_PI * (cp[i].ft * t / T + cp[i].fh * h / H + cp[i].fw * w / W) +
                               cp[i].phi);
                double x[MAX_D];
                double ss = 0.0;
                for (int c = 0; c < d; c += 2) {
                    /* d is even: elements c, c+1 are the two outputs of one
                     * Box-Muller pair; this equals ctr_normal(nkey, tok*d+c+e). */
                    const uint64_t pair = ((uint64_t)tok * d + c) >> 1;
                    const double u1 = 1.0 - ctr_u01(nkey, 2 * pair);
                    const double u2 = ctr_u01(nkey, 2 * pair + 1);
                    const double r = sqrt(-2.0 * log(u1));
                    const double a = 2.0 * M_PI * u2;
                    const double nz[2] = {r * cos(a), r * sin(a)};
                    for (int e = 0; e < 2; ++e) {
                        double v = 0.3 * nz[e];
                        for (int i = 0; i < NCOMP; ++i) v += cp[i].u[c + e] * s[i];
                        x[c + e] = v;
                        ss += v * v;
                    }
                }
                double inv = rms_norm ? 1.0 / sqrt(ss / d + 1e-6) : 1.0;
                uint16_t* o = base + tok * d;
                for (int c = 0; c < d; ++c) o[c] = f32_to_bf16_rne((float)(x[c] * inv));
            }
        }
    }
    return 0;
}

/* The whole head range of batch elements [b_offset, b_offset + B). */
int synth_field_bf16(uint16_t* out, int B, int b_offset, int heads, int T, int H, int W,
                     int d, uint64_t seed, uint32_t tensor, int rms_norm, double tfreq_mult,
                     int cond_frames, uint64_t cond_seed) {
    return synth_field_bf16_slice(out, B, b_offset, heads, 0, T, H, W, d, seed, tensor, rms_norm,
                                  tfreq_mult, cond_frames, cond_seed);
}

/* Raw access to the counter generator, for tests of the generator itself. */
uint64_t synth_ctr_u64(uint64_t key, uint64_t ctr) { return ctr_u64(key, ctr); }
double synth_ctr_normal(uint64_t key, uint64_t idx) { return ctr_normal(key, idx); }
uint64_t synth_mix64(uint64_t z) { return mix64(z); }
