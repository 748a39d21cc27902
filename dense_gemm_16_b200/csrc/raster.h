// raster.h -- grouped-M ordering of output tiles (host and device).
//
// A linear tile index t over a grid_m x grid_n grid of output tiles is mapped
// so that consecutive indices walk down a band of `group_m` tile rows, one
// tile column at a time, then move to the next band.  Tiles that run at the
// same time then cover a near-square patch of the output and share their A
// row panels and B column panels in L2 ("Triton 学习笔记" section 2.3.7: on a
// 9x9 tile grid, 9 tiles in row-major order read 90 input blocks, in 3x3
// groups only 54; the grouped pid mapping of the Gluon/Triton page's
// matmul example).  The last band may be shorter than group_m.
#pragma once

#ifdef __CUDACC__
#define DG16_HD __host__ __device__ __forceinline__
#else
#define DG16_HD inline
#endif

namespace dg16 {

DG16_HD void raster_tile(long long t, int grid_m, int grid_n, int group_m, int& m, int& n) {
  const long long per_band = static_cast<long long>(group_m) * grid_n;
  const long long band = t / per_band;
  const int first_m = static_cast<int>(band * group_m);
  const int rows = (grid_m - first_m) < group_m ? (grid_m - first_m) : group_m;
  const long long r = t - band * per_band;
  m = first_m + static_cast<int>(r % rows);
  n = static_cast<int>(r / rows);
}

}  // namespace dg16
