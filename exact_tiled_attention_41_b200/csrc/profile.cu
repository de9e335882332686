// profile.cu -- optional CUDA-event timing of the main kernels (fa_profile_begin /
// fa_profile_read in include/fa.h).  Off by default; when on, each recorded
// launch costs two cudaEventRecord calls on the launching stream.
#include "../../include/fa.h"
#include "internal.h"

namespace fa {

namespace {
constexpr int kIds = 5;
constexpr int kMaxRec = 1024;
struct Rec {
    cudaEvent_t start[kMaxRec];
    cudaEvent_t stop[kMaxRec];
    int created = 0;
    int count = 0;
    bool pending = false;
};
bool g_enabled = false;
int g_device = -1;
Rec g_rec[kIds];
}  // namespace

void prof_before(int id, cudaStream_t s) {
    if (!g_enabled || id < 0 || id >= kIds) return;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != g_device) return;
    Rec& r = g_rec[id];
    r.pending = false;
    if (r.count >= kMaxRec) return;
    if (r.count >= r.created) {
        if (cudaEventCreate(&r.start[r.count]) != cudaSuccess) return;
        if (cudaEventCreate(&r.stop[r.count]) != cudaSuccess) {
            cudaEventDestroy(r.start[r.count]);
            return;
        }
        r.created = r.count + 1;
    }
    if (cudaEventRecord(r.start[r.count], s) == cudaSuccess) r.pending = true;
}

void prof_after(int id, cudaStream_t s) {
    if (!g_enabled || id < 0 || id >= kIds) return;
    Rec& r = g_rec[id];
    if (!r.pending) return;
    r.pending = false;
    if (cudaEventRecord(r.stop[r.count], s) == cudaSuccess) ++r.count;
}

}  // namespace fa

using namespace fa;

extern "C" {

int fa_profile_begin(int enable) {
    int dev = -1;
    if (enable && cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (enable && g_device != -1 && dev != g_device) {
        // events belong to the device they were created on
        for (auto& r : g_rec) {
            for (int i = 0; i < r.created; ++i) {
                cudaEventDestroy(r.start[i]);
                cudaEventDestroy(r.stop[i]);
            }
            r.created = 0;
        }
    }
    if (enable) {
        // a new recording session starts empty; stopping keeps the records for fa_profile_read
        for (auto& r : g_rec) {
            r.count = 0;
            r.pending = false;
        }
        g_device = dev;
    }
    g_enabled = enable != 0;
    return FA_OK;
}

int fa_profile_read(int kernel_id, int* launches, float* total_ms) {
    if (kernel_id < 0 || kernel_id >= kIds || launches == nullptr || total_ms == nullptr) return FA_ERR_INVALID_ARG;
    const Rec& r = g_rec[kernel_id];
    float tot = 0.f;
    for (int i = 0; i < r.count; ++i) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.start[i], r.stop[i]) != cudaSuccess) return FA_ERR_CUDA;
        tot += ms;
    }
    *launches = r.count;
    *total_ms = tot;
    return FA_OK;
}

}  // extern "C"
