// Pose path front (PersonaLive write-up, "三条条件通路": pose as a residual):
// retargeting of the 21 implicit keypoints (the reference's canonical points
// and scale, the driving frame's rotation, half its translation), the
// prefill ramp of keypoints, and the dot image of 7 selected points that the
// pose guider would take as input.
//
// Keypoints and pixel tests are fp64 with every rounding spelled out (no
// fused multiply-add), so which pixels a dot covers is decided exactly as a
// plain left-to-right evaluation decides it.
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/pl.h"

namespace {

constexpr int kPoints = PL_POSE_POINTS;   // 21 implicit keypoints
constexpr int kDots = PL_POSE_DOTS;       // 7 drawn

struct DotParams {
  int sel[kDots];
  float colour[kDots][3];
};

// kps[f][j] = scale * R(pose_f) c[sel_j] + 0.5 t_f, R = Rz(roll) Ry(yaw) Rx(pitch)
__global__ void pose_keypoints_kernel(const float* __restrict__ canon, float scale,
                                      const float* __restrict__ poses, int frames, DotParams dp,
                                      double* __restrict__ kps) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= frames) return;
  const float* ps = poses + 6 * f;
  const double deg = 3.141592653589793 / 180.0;
  double sp, cp, sy, cy, sr, cr;
  sincos(__dmul_rn(static_cast<double>(ps[0]), deg), &sp, &cp);
  sincos(__dmul_rn(static_cast<double>(ps[1]), deg), &sy, &cy);
  sincos(__dmul_rn(static_cast<double>(ps[2]), deg), &sr, &cr);
  // Rz Ry Rx, row by row
  const double R[3][3] = {
      {__dmul_rn(cr, cy), __dsub_rn(__dmul_rn(__dmul_rn(cr, sy), sp), __dmul_rn(sr, cp)),
       __dadd_rn(__dmul_rn(__dmul_rn(cr, sy), cp), __dmul_rn(sr, sp))},
      {__dmul_rn(sr, cy), __dadd_rn(__dmul_rn(__dmul_rn(sr, sy), sp), __dmul_rn(cr, cp)),
       __dsub_rn(__dmul_rn(__dmul_rn(sr, sy), cp), __dmul_rn(cr, sp))},
      {-sy, __dmul_rn(cy, sp), __dmul_rn(cy, cp)}};
  for (int j = 0; j < kDots; ++j) {
    const float* c = canon + 3 * dp.sel[j];
    for (int a = 0; a < 3; ++a) {
      double acc = __dmul_rn(R[a][0], static_cast<double>(c[0]));
      acc = __dadd_rn(acc, __dmul_rn(R[a][1], static_cast<double>(c[1])));
      acc = __dadd_rn(acc, __dmul_rn(R[a][2], static_cast<double>(c[2])));
      kps[(static_cast<int64_t>(f) * kDots + j) * 3 + a] =
          __dadd_rn(__dmul_rn(static_cast<double>(scale), acc),
                    __dmul_rn(0.5, static_cast<double>(ps[3 + a])));
    }
  }
}

// out[k] = a + (k / frames) (b - a), k < frames (the ramp's last point dropped)
__global__ void pose_ramp_kernel(const double* __restrict__ a, const double* __restrict__ b,
                                 int frames, double* __restrict__ out) {
  const int n = kDots * 3;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= frames * n) return;
  const int k = i / n, e = i - k * n;
  const double w = static_cast<double>(k) / static_cast<double>(frames);
  out[i] = __dadd_rn(a[e], __dmul_rn(w, __dsub_rn(b[e], a[e])));
}

// image[f][ch][y][x] = colour of the last dot covering pixel centre (x+.5, y+.5)
__global__ void pose_dots_kernel(const double* __restrict__ kps, int frames, DotParams dp,
                                 double r2, int H, int W, float* __restrict__ image) {
  const int f = blockIdx.z;
  __shared__ double cx[kDots], cy[kDots];
  __shared__ float fx[kDots], fy[kDots];
  if (threadIdx.x < kDots) {
    const double* k = kps + (static_cast<int64_t>(f) * kDots + threadIdx.x) * 3;
    cx[threadIdx.x] = __dmul_rn(__dmul_rn(__dadd_rn(k[0], 1.0), 0.5), static_cast<double>(W));
    cy[threadIdx.x] = __dmul_rn(__dmul_rn(__dadd_rn(k[1], 1.0), 0.5), static_cast<double>(H));
    fx[threadIdx.x] = static_cast<float>(cx[threadIdx.x]);
    fy[threadIdx.x] = static_cast<float>(cy[threadIdx.x]);
  }
  __syncthreads();
  // a pixel farther than radius + 1 from a centre in either axis (fp32, far
  // beyond its rounding) cannot pass the exact test: skip the fp64 work there
  const float reach = static_cast<float>(sqrt(r2)) + 1.f;
  const int64_t plane = static_cast<int64_t>(H) * W;
  float* img = image + static_cast<int64_t>(f) * 3 * plane;
  // plane < 2^31 (checked on the host): 32-bit pixel indices and division
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < plane; p += gridDim.x * blockDim.x) {
    const int y = p / W, x = p - y * W;
    const double px = x + 0.5, py = y + 0.5;
    int hit = -1;
#pragma unroll
    for (int j = 0; j < kDots; ++j) {
      if (fabsf(static_cast<float>(px) - fx[j]) > reach ||
          fabsf(static_cast<float>(py) - fy[j]) > reach)
        continue;
      const double dx = __dsub_rn(px, cx[j]), dy = __dsub_rn(py, cy[j]);
      if (__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)) <= r2) hit = j;
    }
    img[p] = hit < 0 ? 0.f : dp.colour[hit][0];
    img[plane + p] = hit < 0 ? 0.f : dp.colour[hit][1];
    img[2 * plane + p] = hit < 0 ? 0.f : dp.colour[hit][2];
  }
}

}  // namespace

extern "C" {

pl_status pl_pose_keypoints(const float* canon, float scale, const float* poses, int frames,
                            const int32_t* sel, double* kps, void* stream) {
  if (!canon || !poses || !sel || !kps || frames < 1 || frames > (1 << 24)) return PL_EINVAL;
  if (!std::isfinite(scale)) return PL_EINVAL;
  DotParams dp{};
  for (int j = 0; j < kDots; ++j) {
    if (sel[j] < 0 || sel[j] >= kPoints) return PL_EINVAL;
    dp.sel[j] = sel[j];
  }
  pose_keypoints_kernel<<<(frames + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      canon, scale, poses, frames, dp, kps);
  return cudaGetLastError() == cudaSuccess ? PL_OK : PL_ECUDA;
}

pl_status pl_pose_ramp(const double* kps_from, const double* kps_to, int frames, double* out,
                       void* stream) {
  if (!kps_from || !kps_to || !out || frames < 1 || frames > (1 << 20)) return PL_EINVAL;
  const int n = frames * kDots * 3;
  pose_ramp_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      kps_from, kps_to, frames, out);
  return cudaGetLastError() == cudaSuccess ? PL_OK : PL_ECUDA;
}

pl_status pl_pose_dots(const double* kps, int frames, const float* colours, float radius, int H,
                       int W, float* image, void* stream) {
  if (!kps || !colours || !image || frames < 1 || frames > 65535) return PL_EINVAL;
  if (H < 1 || W < 1 || static_cast<int64_t>(H) * W >= (1ll << 31) - 65536) return PL_EINVAL;
  if (!(radius >= 0.f) || !std::isfinite(radius)) return PL_EINVAL;
  DotParams dp{};
  for (int j = 0; j < kDots; ++j)
    for (int c = 0; c < 3; ++c) dp.colour[j][c] = colours[3 * j + c];
  // about 8 blocks per SM in all, so each thread covers many pixels and the
  // per-block set-up (the 7 centres) is paid rarely
  const int64_t plane = static_cast<int64_t>(H) * W;
  int64_t bx = (plane + 255) / 256;
  const int64_t cap = (148 * 8 + frames - 1) / frames;
  if (bx > cap) bx = cap;
  const double r = radius;
  const dim3 grid(static_cast<unsigned>(bx), 1, frames);
  pose_dots_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(kps, frames, dp, r * r, H,
                                                                       W, image);
  return cudaGetLastError() == cudaSuccess ? PL_OK : PL_ECUDA;
}

}  // extern "C"
