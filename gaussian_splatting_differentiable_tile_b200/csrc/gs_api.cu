// gs_api.cu -- the extern "C" entry points declared in include/gs.h:
// argument checks, buffer carving, launches, status readback, profiling.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "gs_internal.cuh"

using namespace gs;

namespace {

constexpr int64_t kMaxCount = (int64_t(1) << 30) - 1;  // N and max_pairs limit

inline bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

int make_cam(const gs_camera *cam, CamConst *out) {
    if (!cam) return GS_ERR_INVALID_ARG;
    if (cam->width < 1 || cam->height < 1 || cam->width > 65536 || cam->height > 65536)
        return GS_ERR_INVALID_ARG;
    if (!(cam->fx > 0.f) || !(cam->fy > 0.f) || !std::isfinite(cam->fx) || !std::isfinite(cam->fy) ||
        !std::isfinite(cam->cx) || !std::isfinite(cam->cy) || !(cam->near_z > 0.f) ||
        !std::isfinite(cam->near_z))
        return GS_ERR_INVALID_ARG;
    for (int k = 0; k < 16; k++)
        if (!std::isfinite(cam->viewmat[k])) return GS_ERR_INVALID_ARG;
    for (int k = 0; k < 3; k++)
        if (!std::isfinite(cam->bg[k])) return GS_ERR_INVALID_ARG;
    if (cam->flags & ~GS_FLAGS_ALL) return GS_ERR_INVALID_ARG;
    CamConst c{};
    for (int i = 0; i < 3; i++) {
        for (int j = 0; j < 3; j++) c.R[3 * i + j] = cam->viewmat[4 * i + j];
        c.t[i] = cam->viewmat[4 * i + 3];
    }
    c.fx = cam->fx; c.fy = cam->fy; c.cx = cam->cx; c.cy = cam->cy;
    // "Gaussian splatting in PyTorch" s3: frustum widened by 0.3 of the
    // half-FoV tangent on each side (computed in double, rounded once).
    const double tfx = 0.5 * cam->width / (double)cam->fx, tfy = 0.5 * cam->height / (double)cam->fy;
    c.lim_x_lo = (float)(-((double)cam->cx / cam->fx + 0.3 * tfx));
    c.lim_x_hi = (float)((cam->width - (double)cam->cx) / cam->fx + 0.3 * tfx);
    c.lim_y_lo = (float)(-((double)cam->cy / cam->fy + 0.3 * tfy));
    c.lim_y_hi = (float)((cam->height - (double)cam->cy) / cam->fy + 0.3 * tfy);
    c.near_z = cam->near_z;
    for (int k = 0; k < 3; k++) c.bg[k] = cam->bg[k];
    c.width = cam->width;
    c.height = cam->height;
    c.tiles_x = (cam->width + kTile - 1) / kTile;
    c.tiles_y = (cam->height + kTile - 1) / kTile;
    c.flags = cam->flags;
    // [GSP] s5/s6: alpha cap 0.99 (3DGS) or 0.999 (older gsplat); the stop
    // test next_T < 1e-4 (3DGS) or <= 1e-4 (gsplat), the latter as
    // next_T < the float after 1e-4.
    c.alpha_cap = (cam->flags & GS_FLAG_CAP_0999) ? 0.999f : 0.99f;
    c.t_stop = (cam->flags & GS_FLAG_STOP_INCLUSIVE) ? std::nextafter(1e-4f, 1.f) : 1e-4f;
    *out = c;
    return GS_OK;
}

int check_projected(const gs_projected *p, int64_t n) {
    if (!p) return GS_ERR_INVALID_ARG;
    if (n == 0) return GS_OK;
    if (!p->xy_opacity_depth || !p->conic_radius || !p->rgb || !p->rect || !p->count)
        return GS_ERR_INVALID_ARG;
    if (!aligned(p->xy_opacity_depth, 16) || !aligned(p->conic_radius, 16) || !aligned(p->rgb, 16) ||
        !aligned(p->rect, 16) || !aligned(p->count, 4))
        return GS_ERR_ALIGNMENT;
    return GS_OK;
}

int check_params(const gs_params *p, int64_t n) {
    if (!p) return GS_ERR_INVALID_ARG;
    if (n == 0) return GS_OK;
    if (!p->means || !p->log_scales || !p->quats || !p->opacity_logits || !p->colors)
        return GS_ERR_INVALID_ARG;
    if (!aligned(p->means, 4) || !aligned(p->log_scales, 4) || !aligned(p->quats, 16) ||
        !aligned(p->opacity_logits, 4) || !aligned(p->colors, 4))
        return GS_ERR_ALIGNMENT;
    return GS_OK;
}

int check_bins(const gs_bins *b, int64_t n, const CamConst &c, BinsLayout *L) {
    if (!b || !b->scratch || !b->pair_tile || !b->pair_gid || !b->ranges || !b->n_pairs || !b->status)
        return GS_ERR_INVALID_ARG;
    if (n > b->max_n || (int64_t)c.tiles_x * c.tiles_y > b->max_tiles) return GS_ERR_INVALID_ARG;
    if (b->max_n < 0 || b->max_pairs < 0 || b->max_n > kMaxCount || b->max_pairs > kMaxCount)
        return GS_ERR_TOO_LARGE;
    if (b->strategy < GS_BIN_AUTO || b->strategy > GS_BIN_GLOBAL) return GS_ERR_INVALID_ARG;
    *L = bins_layout(b->max_n, b->max_pairs, b->max_tiles);
    if (b->scratch_bytes < L->total || !aligned(b->scratch, 256)) return GS_ERR_INVALID_ARG;
    return GS_OK;
}

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// ---------------------------------------------------------------- profiling
struct ProfRec {
    const char *name;
    cudaEvent_t a, b;
    int kernels;  // kernel launches between the two events
};
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_pool;
bool g_prof_on = false;
bool g_prof_pending = false;
int32_t g_prof_max = 0;

cudaEvent_t pool_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

namespace gs {
void prof_before(const char *name, cudaStream_t s) {
    g_prof_pending = false;
    if (!g_prof_on || (int32_t)g_prof.size() >= g_prof_max) return;
    ProfRec r{name, pool_event(), pool_event(), 1};
    if (!r.a || !r.b) return;
    cudaEventRecord(r.a, s);
    g_prof.push_back(r);
    g_prof_pending = true;
}
void prof_after(cudaStream_t s, int kernels) {
    if (!g_prof_pending) return;
    g_prof.back().kernels = kernels;
    cudaEventRecord(g_prof.back().b, s);
    g_prof_pending = false;
}
}  // namespace gs

extern "C" {

int gs_version(void) { return 1; }

const char *gs_error_string(int code) {
    switch (code) {
        case GS_OK: return "ok";
        case GS_ERR_INVALID_ARG: return "invalid argument (size, pointer or camera value out of range)";
        case GS_ERR_CAPACITY: return "pair list exceeds max_pairs: regrow the bins buffer and retry";
        case GS_ERR_TOO_LARGE: return "N or max_pairs at or above 2^30";
        case GS_ERR_ALIGNMENT: return "pointer not aligned as documented";
        case GS_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case GS_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
        case GS_ERR_BOUNDS: return "a kernel index was out of range and its access skipped (checked build)";
        default: return "unknown error code";
    }
}

size_t gs_projected_bytes(int64_t n) {
    if (n < 0) return 0;
    const size_t v4 = align_up((size_t)n * 16, 256);
    return 4 * v4 + align_up((size_t)n * 4, 256);
}

int gs_projected_carve(void *base, int64_t n, gs_projected *out) {
    if (!out || n < 0 || (n > 0 && !base)) return GS_ERR_INVALID_ARG;
    if (n > kMaxCount) return GS_ERR_TOO_LARGE;
    if (!aligned(base, 256)) return GS_ERR_ALIGNMENT;
    char *b = static_cast<char *>(base);
    const size_t v4 = align_up((size_t)n * 16, 256);
    out->xy_opacity_depth = reinterpret_cast<float *>(b);
    out->conic_radius = reinterpret_cast<float *>(b + v4);
    out->rgb = reinterpret_cast<float *>(b + 2 * v4);
    out->rect = reinterpret_cast<int32_t *>(b + 3 * v4);
    out->count = reinterpret_cast<uint32_t *>(b + 4 * v4);
    return GS_OK;
}

size_t gs_bins_bytes(int64_t n, int64_t max_pairs, int32_t width, int32_t height) {
    if (n < 0 || max_pairs < 0 || width < 1 || height < 1) return 0;
    const int32_t tiles = ((width + kTile - 1) / kTile) * ((height + kTile - 1) / kTile);
    return bins_layout(n, max_pairs, tiles).total;
}

int gs_bins_carve(void *base, int64_t n, int64_t max_pairs, int32_t width, int32_t height,
                  gs_bins *out) {
    if (!out || !base || n < 0 || max_pairs < 0 || width < 1 || height < 1 || width > 65536 ||
        height > 65536)
        return GS_ERR_INVALID_ARG;
    if (n > kMaxCount || max_pairs > kMaxCount) return GS_ERR_TOO_LARGE;
    if (!aligned(base, 256)) return GS_ERR_ALIGNMENT;
    const int32_t tiles = ((width + kTile - 1) / kTile) * ((height + kTile - 1) / kTile);
    const BinsLayout L = bins_layout(n, max_pairs, tiles);
    char *b = static_cast<char *>(base);
    std::memset(out, 0, sizeof(*out));
    out->pair_tile = reinterpret_cast<uint32_t *>(b + L.pair_tile);
    out->pair_gid = reinterpret_cast<uint32_t *>(b + L.pair_gid);
    out->ranges = reinterpret_cast<uint32_t *>(b + L.ranges);
    out->n_pairs = reinterpret_cast<uint64_t *>(b + L.n_pairs);
    out->status = reinterpret_cast<int32_t *>(b + L.status);
    out->max_pairs = max_pairs;
    out->max_n = n;
    out->max_tiles = tiles;
    out->scratch = base;
    out->scratch_bytes = L.total;
    return GS_OK;
}

int gs_project(const gs_camera *cam, int64_t n, const gs_params *params, const gs_projected *out,
               void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    if (n > kMaxCount) return GS_ERR_TOO_LARGE;
    if ((rc = check_params(params, n)) || (rc = check_projected(out, n))) return rc;
    return launch_project(c, n, *params, *out, as_stream(stream)) == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}

int gs_read_status(const gs_bins *bins, int64_t *n_pairs_host, void *stream) {
    if (!bins || !bins->status || !bins->n_pairs) return GS_ERR_INVALID_ARG;
    int32_t st = 0;
    uint64_t k = 0;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(&st, bins->status, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(&k, bins->n_pairs, sizeof(k), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return GS_ERR_CUDA;
    if (n_pairs_host) *n_pairs_host = (int64_t)k;
    return st;
}

int gs_last_device_error(const gs_bins *bins, void *stream) { return gs_read_status(bins, nullptr, stream); }

size_t gs_sort_bytes(int64_t max_pairs, int32_t tiles) {
    if (max_pairs < 0 || tiles < 1) return 0;
    return bins_layout(0, max_pairs, tiles).total;
}

int gs_bin_and_sort(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                    int64_t *n_pairs_host, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    if (n > kMaxCount) return GS_ERR_TOO_LARGE;
    BinsLayout L;
    if ((rc = check_projected(proj, n)) || (rc = check_bins(bins, n, c, &L))) return rc;
    if (launch_bin_and_sort(c, n, *proj, *bins, L, as_stream(stream)) != cudaSuccess) return GS_ERR_CUDA;
    if (!n_pairs_host) return GS_OK;
    rc = gs_read_status(bins, n_pairs_host, stream);
    if (rc == GS_OK && *n_pairs_host > bins->max_pairs) rc = GS_ERR_CAPACITY;
    return rc;
}

int gs_render_fwd(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                  float *image, float *T_final, uint32_t *last, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_projected(proj, n)) || (rc = check_bins(bins, n, c, &L))) return rc;
    if (!image || !T_final || !last) return GS_ERR_INVALID_ARG;
    if (!aligned(image, 4) || !aligned(T_final, 4) || !aligned(last, 4)) return GS_ERR_ALIGNMENT;
    return launch_render_fwd(c, n, *proj, *bins, image, T_final, last, as_stream(stream)) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_render_fwd_l1(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                     float *image, float *T_final, uint32_t *last, const float *target, float *dL_dimage,
                     float *loss, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_projected(proj, n)) || (rc = check_bins(bins, n, c, &L))) return rc;
    if (!image || !T_final || !last || !target || !dL_dimage) return GS_ERR_INVALID_ARG;
    if (!aligned(image, 4) || !aligned(T_final, 4) || !aligned(last, 4) || !aligned(target, 4) ||
        !aligned(dL_dimage, 4) || (loss && !aligned(loss, 4)))
        return GS_ERR_ALIGNMENT;
    return launch_render_fwd(c, n, *proj, *bins, image, T_final, last, as_stream(stream), target, dL_dimage,
                             loss) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_render_bwd(const gs_camera *cam, int64_t n, const gs_params *params,
                  const gs_projected *proj, const gs_bins *bins, const float *T_final,
                  const uint32_t *last, const float *dL_dimage, float *grad2d,
                  const gs_grads *grads, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_params(params, n)) || (rc = check_projected(proj, n)) ||
        (rc = check_bins(bins, n, c, &L)))
        return rc;
    if (!T_final || !last || !dL_dimage || !grads) return GS_ERR_INVALID_ARG;
    if (n > 0 && (!grad2d || !grads->means || !grads->log_scales || !grads->quats ||
                  !grads->opacity_logits || !grads->colors))
        return GS_ERR_INVALID_ARG;
    if (!aligned(grad2d, 16) || !aligned(grads->quats, 16) || !aligned(T_final, 4) ||
        !aligned(last, 4) || !aligned(dL_dimage, 4))
        return GS_ERR_ALIGNMENT;
    cudaStream_t s = as_stream(stream);
    if (n > 0 && cudaMemsetAsync(grad2d, 0, (size_t)n * 12 * sizeof(float), s) != cudaSuccess)
        return GS_ERR_CUDA;
    if (launch_render_bwd(c, n, *proj, *bins, T_final, last, dL_dimage, grad2d, s) != cudaSuccess)
        return GS_ERR_CUDA;
    if (launch_project_bwd(c, n, *params, *proj, grad2d, *grads, s) != cudaSuccess) return GS_ERR_CUDA;
    return GS_OK;
}

namespace {
constexpr int32_t kMaxFeatures = 1024;
}

int gs_render_features_fwd(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                           const float *features, int32_t F, float *out, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0 || F < 4 || F > kMaxFeatures || F % 4 != 0 || !out || (n > 0 && !features))
        return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_projected(proj, n)) || (rc = check_bins(bins, n, c, &L))) return rc;
    if (!aligned(features, 16) || !aligned(out, 4)) return GS_ERR_ALIGNMENT;
    return launch_render_features_fwd(c, n, *proj, *bins, features, F, out, as_stream(stream)) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_render_features_bwd(const gs_camera *cam, int64_t n, const gs_params *params, const gs_projected *proj,
                           const gs_bins *bins, const float *T_final, const uint32_t *last,
                           const float *features, int32_t F, const float *dL_dout, float *grad2d,
                           float *dL_dfeatures, const gs_grads *grads, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0 || F < 4 || F > kMaxFeatures || F % 4 != 0) return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_params(params, n)) || (rc = check_projected(proj, n)) ||
        (rc = check_bins(bins, n, c, &L)))
        return rc;
    if (!T_final || !last || !dL_dout || !grads) return GS_ERR_INVALID_ARG;
    if (n > 0 && (!features || !grad2d || !dL_dfeatures || !grads->means || !grads->log_scales ||
                  !grads->quats || !grads->opacity_logits || !grads->colors))
        return GS_ERR_INVALID_ARG;
    if (!aligned(features, 16) || !aligned(grad2d, 16) || !aligned(grads->quats, 16) || !aligned(T_final, 4) ||
        !aligned(last, 4) || !aligned(dL_dout, 4) || !aligned(dL_dfeatures, 4))
        return GS_ERR_ALIGNMENT;
    if (n == 0) return GS_OK;
    cudaStream_t s = as_stream(stream);
    if (cudaMemsetAsync(grad2d, 0, (size_t)n * 12 * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(dL_dfeatures, 0, (size_t)n * F * sizeof(float), s) != cudaSuccess)
        return GS_ERR_CUDA;
    if (launch_render_features_bwd(c, n, *proj, *bins, T_final, last, features, F, dL_dout, grad2d, dL_dfeatures,
                                   s) != cudaSuccess)
        return GS_ERR_CUDA;
    // the features' share of dL/d(mean2d, conic, opacity), added into grads
    if (launch_project_bwd(c, n, *params, *proj, grad2d, *grads, s, true) != cudaSuccess) return GS_ERR_CUDA;
    return GS_OK;
}

int gs_render_stats(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                    const uint32_t *last, uint64_t *counts, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0) return GS_ERR_INVALID_ARG;
    BinsLayout L;
    if ((rc = check_projected(proj, n)) || (rc = check_bins(bins, n, c, &L))) return rc;
    if (!last || !counts) return GS_ERR_INVALID_ARG;
    if (!aligned(last, 4) || !aligned(counts, 8)) return GS_ERR_ALIGNMENT;
    return launch_render_stats(c, n, *proj, *bins, last, counts, as_stream(stream)) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_l1_loss_grad(const float *image, const float *target, int64_t count, float *dL_dimage,
                    float *loss, void *stream) {
    if (count < 0 || (count > 0 && (!image || !target || !dL_dimage))) return GS_ERR_INVALID_ARG;
    return launch_l1(image, target, count, dL_dimage, loss, as_stream(stream)) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

// ---------------------------------------------------------------- training
namespace {

bool set_complete(const gs_param_set *p) {
    return p && p->means && p->log_scales && p->quats && p->opacity_logits && p->colors;
}

int check_adam_cfg(const gs_adam_config *cfg) {
    if (!cfg) return GS_ERR_INVALID_ARG;
    for (float lr : cfg->lr)
        if (!std::isfinite(lr) || lr < 0.f) return GS_ERR_INVALID_ARG;
    if (!(cfg->beta1 >= 0.0 && cfg->beta1 < 1.0) || !(cfg->beta2 >= 0.0 && cfg->beta2 < 1.0) ||
        !(cfg->eps > 0.f) || !std::isfinite(cfg->eps))
        return GS_ERR_INVALID_ARG;
    return GS_OK;
}

AdamBetas adam_betas(const gs_adam_config *cfg) {
    AdamBetas b{};
    if (!cfg) return b;
    b.b1 = cfg->beta1;
    b.b2 = cfg->beta2;
    b.b1f = (float)cfg->beta1;
    b.b2f = (float)cfg->beta2;
    b.omb1 = (float)(1.0 - cfg->beta1);
    b.omb2 = (float)(1.0 - cfg->beta2);
    return b;
}

// Adam's launch description from the parameter, moment, slot and output sets.
// M and V are null for a gradient sum without update.
int adam_groups(int64_t n, const gs_param_set &P, const gs_param_set *slots, int n_slots,
                const gs_param_set *M, const gs_param_set *V, const gs_param_set *out,
                const gs_adam_config *cfg, AdamGroups *G) {
    float *gs_param_set::*field[5] = {&gs_param_set::means, &gs_param_set::log_scales, &gs_param_set::quats,
                                      &gs_param_set::opacity_logits, &gs_param_set::colors};
    const int64_t width[5] = {3, 3, 4, 1, 3};
    for (int k = 0; k < 5; k++) {
        AdamGroup &A = G->g[k];
        A = AdamGroup{};
        A.p = P.*field[k];
        A.m = M ? M->*field[k] : nullptr;
        A.v = V ? V->*field[k] : nullptr;
        A.out = out ? out->*field[k] : nullptr;
        A.count = n * width[k];
        A.lr = cfg ? cfg->lr[k] : 0.f;
        bool vec = aligned(A.p, 16) && aligned(A.m, 16) && aligned(A.v, 16) && aligned(A.out, 16);
        for (int s = 0; s < n_slots; s++) {
            A.slot[s] = slots[s].*field[k];
            vec = vec && aligned(A.slot[s], 16);
        }
        A.vec = vec ? 1 : 0;
        if (k == 2 && !vec) return GS_ERR_ALIGNMENT;  // quaternion arrays are float4
        if (!aligned(A.p, 4) || !aligned(A.m, 4) || !aligned(A.v, 4) || !aligned(A.out, 4))
            return GS_ERR_ALIGNMENT;
        for (int s = 0; s < n_slots; s++)
            if (!aligned(A.slot[s], 4)) return GS_ERR_ALIGNMENT;
    }
    return GS_OK;
}

}  // namespace

int gs_adam_step(int64_t n, const gs_param_set *params, const gs_param_set *slots, int32_t n_slots,
                 float grad_scale, const gs_param_set *m, const gs_param_set *v,
                 const gs_adam_config *cfg, int64_t *step, const gs_param_set *grad_out,
                 void *stream) {
    if (n < 0 || n_slots < 1 || n_slots > kAdamMaxSlots || !step || !params || !slots || !m || !v ||
        !std::isfinite(grad_scale))
        return GS_ERR_INVALID_ARG;
    if (n > kMaxCount) return GS_ERR_TOO_LARGE;
    int rc = check_adam_cfg(cfg);
    if (rc) return rc;
    if (!aligned(step, 8)) return GS_ERR_ALIGNMENT;
    if (n > 0) {
        if (!set_complete(params) || !set_complete(m) || !set_complete(v) ||
            (grad_out && !set_complete(grad_out)))
            return GS_ERR_INVALID_ARG;
        for (int s = 0; s < n_slots; s++)
            if (!set_complete(&slots[s])) return GS_ERR_INVALID_ARG;
    }
    AdamGroups G;
    if (n > 0 && (rc = adam_groups(n, *params, slots, n_slots, m, v, grad_out, cfg, &G))) return rc;
    return launch_adam(G, n > 0 ? 4 * n : 0, adam_betas(cfg), cfg->eps, grad_scale, n_slots, step,
                       as_stream(stream)) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_train_step(const gs_camera *cams, int32_t n_cams, int64_t n, const gs_param_set *params,
                  const float *targets, const gs_train_lane *lanes, int32_t n_lanes, void *fork,
                  const gs_param_set *m, const gs_param_set *v, const gs_adam_config *cfg,
                  int64_t *step, float *losses, int64_t *cam_stats, const gs_param_set *grad_out,
                  void *stream) {
    if (!cams || n_cams < 1 || !lanes || n_lanes < 1 || n_lanes > kAdamMaxSlots || n < 0 || !params ||
        !targets)
        return GS_ERR_INVALID_ARG;
    if (n > kMaxCount) return GS_ERR_TOO_LARGE;
    if (!cfg && !grad_out) return GS_ERR_INVALID_ARG;
    int rc;
    if (cfg && ((rc = check_adam_cfg(cfg)) || !m || !v || !step)) return rc ? rc : GS_ERR_INVALID_ARG;
    if (cfg && !aligned(step, 8)) return GS_ERR_ALIGNMENT;
    if (!aligned(targets, 4) || (losses && !aligned(losses, 4)) || (cam_stats && !aligned(cam_stats, 8)))
        return GS_ERR_ALIGNMENT;
    if (n > 0 && (!set_complete(params) || (cfg && (!set_complete(m) || !set_complete(v))) ||
                  (grad_out && !set_complete(grad_out))))
        return GS_ERR_INVALID_ARG;
    // cameras: valid, one image size and channel count
    std::vector<CamConst> cc((size_t)n_cams);
    for (int b = 0; b < n_cams; b++) {
        if ((rc = make_cam(&cams[b], &cc[b]))) return rc;
        if (cc[b].width != cc[0].width || cc[b].height != cc[0].height ||
            ((cc[b].flags ^ cc[0].flags) & GS_FLAG_DEPTH))
            return GS_ERR_INVALID_ARG;
    }
    const int64_t pixels = (int64_t)cc[0].width * cc[0].height;
    const int64_t values = pixels * ((cc[0].flags & GS_FLAG_DEPTH) ? 4 : 3);
    gs_params pc{params->means, params->log_scales, params->quats, params->opacity_logits, params->colors};
    if ((rc = check_params(&pc, n))) return rc;
    // lanes: complete buffers for this camera size and N
    const int used = std::min(n_lanes, n_cams);
    std::vector<BinsLayout> L((size_t)used);
    for (int l = 0; l < used; l++) {
        const gs_train_lane &ln = lanes[l];
        if ((rc = check_projected(&ln.proj, n)) || (rc = check_bins(&ln.bins, n, cc[0], &L[l]))) return rc;
        if (!ln.image || !ln.T_final || !ln.last || !ln.dL_dimage || (n > 0 && !ln.grad2d))
            return GS_ERR_INVALID_ARG;
        if (n > 0 && !set_complete(&ln.grads)) return GS_ERR_INVALID_ARG;
        if (!aligned(ln.image, 4) || !aligned(ln.T_final, 4) || !aligned(ln.last, 4) ||
            !aligned(ln.dL_dimage, 4) || !aligned(ln.grad2d, 16) || !aligned(ln.grads.quats, 16))
            return GS_ERR_ALIGNMENT;
        if (ln.stream != stream && (!fork || !ln.done)) return GS_ERR_INVALID_ARG;
    }
    // the Adam (or gradient-sum) launch is described before anything runs
    std::vector<gs_param_set> slots((size_t)used);
    for (int l = 0; l < used; l++) slots[l] = lanes[l].grads;
    AdamGroups G;
    if (n > 0 && (rc = adam_groups(n, *params, slots.data(), used, cfg ? m : nullptr, cfg ? v : nullptr,
                                   grad_out, cfg, &G)))
        return rc;

    cudaStream_t s = as_stream(stream);
    bool forked = false;
    for (int l = 0; l < used; l++)
        if (lanes[l].stream != stream) forked = true;
    if (forked && cudaEventRecord(reinterpret_cast<cudaEvent_t>(fork), s) != cudaSuccess) return GS_ERR_CUDA;
    for (int l = 0; l < used; l++) {
        const gs_train_lane &ln = lanes[l];
        cudaStream_t ls = as_stream(ln.stream);
        if (ln.stream != stream && cudaStreamWaitEvent(ls, reinterpret_cast<cudaEvent_t>(fork), 0) != cudaSuccess)
            return GS_ERR_CUDA;
        for (int b = l; b < n_cams; b += n_lanes) {
            const CamConst &c = cc[b];
            const gs_params &pp = pc;
            if (launch_project(c, n, pp, ln.proj, ls) != cudaSuccess ||
                launch_bin_and_sort(c, n, ln.proj, ln.bins, L[l], ls) != cudaSuccess ||
                launch_render_fwd(c, n, ln.proj, ln.bins, ln.image, ln.T_final, ln.last, ls,
                                  targets + (size_t)b * values, ln.dL_dimage, losses ? losses + b : nullptr,
                                  cam_stats ? cam_stats + 2 * b : nullptr) != cudaSuccess)
                return GS_ERR_CUDA;
            if (n > 0 && cudaMemsetAsync(ln.grad2d, 0, (size_t)n * 12 * sizeof(float), ls) != cudaSuccess)
                return GS_ERR_CUDA;
            if (launch_render_bwd(c, n, ln.proj, ln.bins, ln.T_final, ln.last, ln.dL_dimage, ln.grad2d, ls) !=
                    cudaSuccess ||
                launch_project_bwd(c, n, pp, ln.proj, ln.grad2d, ln.grads, ls, b >= n_lanes) != cudaSuccess)
                return GS_ERR_CUDA;
        }
        if (ln.stream != stream &&
            (cudaEventRecord(reinterpret_cast<cudaEvent_t>(ln.done), ls) != cudaSuccess ||
             cudaStreamWaitEvent(s, reinterpret_cast<cudaEvent_t>(ln.done), 0) != cudaSuccess))
            return GS_ERR_CUDA;
    }
    const float scale = 1.f / (float)n_cams;
    if (cfg)
        return launch_adam(G, n > 0 ? 4 * n : 0, adam_betas(cfg), cfg->eps, scale, used, step, s) ==
                       cudaSuccess
                   ? GS_OK
                   : GS_ERR_CUDA;
    return launch_adam(G, n > 0 ? 4 * n : 0, adam_betas(nullptr), 1.f, scale, used, nullptr, s, false) == cudaSuccess
               ? GS_OK
               : GS_ERR_CUDA;
}

int gs_profile_begin(int32_t max_launches) {
    if (max_launches < 0) return GS_ERR_INVALID_ARG;
    for (auto &r : g_prof) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_prof.clear();
    g_prof.reserve((size_t)max_launches);
    g_prof_max = max_launches;
    g_prof_on = true;
    g_prof_pending = false;
    return GS_OK;
}

int gs_profile_end(gs_profile_stat *out, int32_t max_stats) {
    g_prof_on = false;
    std::vector<gs_profile_stat> stats;
    int rc = GS_OK;
    for (auto &r : g_prof) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            rc = GS_ERR_CUDA;
            continue;
        }
        gs_profile_stat *hit = nullptr;
        for (auto &s : stats)
            if (std::strncmp(s.name, r.name, sizeof(s.name)) == 0) hit = &s;
        if (!hit) {
            gs_profile_stat s{};
            std::snprintf(s.name, sizeof(s.name), "%s", r.name);
            stats.push_back(s);
            hit = &stats.back();
        }
        hit->launches += r.kernels;
        hit->total_ms += ms;
    }
    for (auto &r : g_prof) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_prof.clear();
    if (rc != GS_OK) return rc;
    const int32_t m = (int32_t)stats.size() < max_stats ? (int32_t)stats.size() : max_stats;
    for (int32_t i = 0; i < m && out; i++) out[i] = stats[i];
    return m;
}

}  // extern "C"

// ------------------------------------------------------------------------
// gs_bin_and_sort_static: the binning scratch of gs_bin_and_sort held in one
// fixed-size device array of this library, for callers that cannot allocate.
namespace {

constexpr int64_t kStaticMaxN = int64_t(1) << 18;       // Gaussians
constexpr int64_t kStaticMaxPairs = int64_t(1) << 20;   // pairs
constexpr int32_t kStaticMaxTiles = 65536;              // tiles
constexpr BinsLayout kStaticLayout = bins_layout(kStaticMaxN, kStaticMaxPairs, kStaticMaxTiles);
// Everything the layout holds before its own result arrays: the variant
// writes its results straight into the caller's arrays.
constexpr size_t kStaticBytes = kStaticLayout.pair_tile;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

// Host-side device address of g_static_scratch, per device.  The array's name
// in host code is only a stand-in for the symbol, never an address a kernel
// may be given.
constexpr int kMaxDevices = 128;
void *g_static_ptr[kMaxDevices] = {};
std::mutex g_static_mutex;

int static_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return GS_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return GS_OK;
}

}  // namespace

extern "C" int gs_bin_and_sort_static(const gs_camera *cam, int64_t n, const gs_projected *proj,
                                      uint32_t *pair_tile, uint32_t *pair_gid, uint32_t *ranges,
                                      int64_t max_pairs, int64_t *n_pairs_host, void *stream) {
    CamConst c;
    int rc = make_cam(cam, &c);
    if (rc) return rc;
    if (n < 0 || max_pairs < 0 || !n_pairs_host || !pair_tile || !pair_gid || !ranges)
        return GS_ERR_INVALID_ARG;
    const int64_t tiles = (int64_t)c.tiles_x * c.tiles_y;
    if (n > kStaticMaxN || max_pairs > kStaticMaxPairs || tiles > kStaticMaxTiles)
        return GS_ERR_TOO_LARGE;
    if ((rc = check_projected(proj, n))) return rc;
    if (!aligned(pair_tile, 4) || !aligned(pair_gid, 4) || !aligned(ranges, 8)) return GS_ERR_ALIGNMENT;
    void *base = nullptr;
    if ((rc = static_scratch(&base))) return rc;
    char *b = static_cast<char *>(base);
    gs_bins bins;
    std::memset(&bins, 0, sizeof(bins));
    bins.pair_tile = pair_tile;
    bins.pair_gid = pair_gid;
    bins.ranges = reinterpret_cast<uint32_t *>(b + kStaticLayout.ranges);
    bins.n_pairs = reinterpret_cast<uint64_t *>(b + kStaticLayout.n_pairs);
    bins.status = reinterpret_cast<int32_t *>(b + kStaticLayout.status);
    bins.max_pairs = max_pairs;
    bins.max_n = kStaticMaxN;
    bins.max_tiles = kStaticMaxTiles;
    bins.scratch = base;
    bins.scratch_bytes = kStaticBytes;
    cudaStream_t s = as_stream(stream);
    // Nothing of the previous call leaks in: the launcher's one memset clears
    // the status word and K, and every other array the stages read (the
    // [CTA][tile] count matrix, the per-tile totals, ranges and tile order,
    // the emitted keys, the long-list sort's ping-pong arrays) is written in
    // full, for every tile or pair of this call, before it is read.
    if (launch_bin_and_sort(c, n, *proj, bins, kStaticLayout, s) != cudaSuccess) return GS_ERR_CUDA;
    if (cudaMemcpyAsync(ranges, bins.ranges, (size_t)tiles * 2 * sizeof(uint32_t),
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return GS_ERR_CUDA;
    rc = gs_read_status(&bins, n_pairs_host, stream);
    if (rc == GS_OK && *n_pairs_host > max_pairs) rc = GS_ERR_CAPACITY;
    return rc;
}
