// nm_api.cu -- status text, sizes, version and the device status word.
#include "nm_internal.cuh"

extern "C" const char* nm_status_string(int status) {
  switch (status) {
    case NM_OK: return "NM_OK";
    case NM_ERR_NULL: return "NM_ERR_NULL: a required pointer is NULL";
    case NM_ERR_SHAPE: return "NM_ERR_SHAPE: bad size or leading dimension";
    case NM_ERR_ALIGN: return "NM_ERR_ALIGN: pointer or row stride not 16-byte aligned";
    case NM_ERR_DTYPE: return "NM_ERR_DTYPE: unsupported element type";
    case NM_ERR_NM: return "NM_ERR_NM: need 1 <= N < M <= 8 (2:4 for compression and the product)";
    case NM_ERR_UNSUPPORTED: return "NM_ERR_UNSUPPORTED: not implemented for these arguments";
    case NM_ERR_CUDA: return "NM_ERR_CUDA: a CUDA runtime or driver call failed";
    case NM_ERR_WORKSPACE: return "NM_ERR_WORKSPACE: workspace missing or too small";
    case NM_ERR_TIMEOUT: return "NM_ERR_TIMEOUT: a bounded device-side wait gave up";
    default: return "unknown nm_status";
  }
}

extern "C" int nm_version(void) { return 1 * 10000 + 0 * 100 + 0; }

extern "C" nm_status nm_sizes(int64_t R, int64_t C, int N, int M, nm_dtype dtype, size_t* values_bytes,
                              size_t* meta_bytes, size_t* meta_sm100_bytes) {
  if (!nm::dtype_ok_int8(dtype)) return NM_ERR_DTYPE;
  if (M < 2 || M > 8 || N < 1 || N >= M) return NM_ERR_NM;
  if (R < 0 || C < 0 || C % M != 0) return NM_ERR_SHAPE;
  const bool two_four = (N == 2 && M == 4);
  if (two_four && C % 8 != 0) return NM_ERR_SHAPE;
  const size_t kept = size_t(R) * size_t(C / M) * size_t(N);
  if (values_bytes) *values_bytes = kept * size_t(nm::esize_of(dtype));
  if (meta_bytes) *meta_bytes = two_four ? kept * 2 / 8 : 0;
  if (meta_sm100_bytes) {
    const size_t rp = size_t((R + 127) / 128 * 128), cp = size_t((C + 127) / 128 * 128);
    *meta_sm100_bytes = two_four ? rp * cp / 8 : 0;
  }
  return NM_OK;
}

