// View analysis: validation of a strided view and its reduction to two
// merged index groups ("DeepGEMM: a recalibration of the compute paradigm",
// §2.2: effective span shape[i] * stride[i]; contiguous segments where
// stride[i] == stride[i+1] * shape[i+1]; §3.2: strides are in bytes; §5.1:
// stride products that overflow must be caught, here as int64 overflow).
#include <algorithm>
#include <cstring>

#include "dg_internal.h"

namespace dg {

int elem_size(int dtype) {
    switch (dtype) {
    case DG_F32: return 4;
    case DG_F16: return 2;
    case DG_BF16: return 2;
    case DG_E4M3: return 1;
    default: return 0;
    }
}

// Drop size-1 dims of [lo, hi) and merge neighbours that form one contiguous
// segment.  Returns the group outermost first.
static Axis merge_group(const dg_view *v, int lo, int hi) {
    Axis a{};
    int64_t size[kMaxDims], stride[kMaxDims];
    int n = 0;
    for (int d = lo; d < hi; ++d) {
        if (v->shape[d] == 1) continue;
        size[n] = v->shape[d];
        stride[n] = v->stride[d];
        ++n;
    }
    // merge from the inside out: dim i folds into i+1 when i steps over all of i+1
    int m = 0;
    int64_t msz[kMaxDims], mst[kMaxDims];
    for (int i = 0; i < n; ++i) {
        if (m > 0 && mst[m - 1] == stride[i] * size[i]) {
            // previous (outer) dim is contiguous with this one: fold it in
            msz[m - 1] *= size[i];
            mst[m - 1] = stride[i];
        } else {
            msz[m] = size[i];
            mst[m] = stride[i];
            ++m;
        }
    }
    a.n = m;
    for (int i = 0; i < m; ++i) {
        a.size[i] = msz[i];
        a.stride[i] = mst[i];
    }
    return a;
}

static bool mul_ok(int64_t a, int64_t b, int64_t *r) { return !__builtin_mul_overflow(a, b, r); }
static bool add_ok(int64_t a, int64_t b, int64_t *r) { return !__builtin_add_overflow(a, b, r); }

static int pow2_align(uint64_t x) {
    // largest power of two dividing x, capped at 16 (x == 0 -> 16)
    if (x == 0) return 16;
    int a = 1;
    while (a < 16 && (x % (uint64_t)(a * 2)) == 0) a *= 2;
    return a;
}

dg_status analyse(const dg_view *v, bool is_output, ViewInfo *info) {
    if (!v || !info) return DG_ERR_NULL;
    if (v->ndim < 1 || v->ndim > kMaxDims || v->row_dims < 0 || v->row_dims > v->ndim) return DG_ERR_NDIM;
    const int es = elem_size(v->dtype);
    if (es == 0) return DG_ERR_DTYPE;
    ViewInfo r;
    r.es = es;
    int64_t rows = 1, cols = 1;
    bool empty = false;
    for (int d = 0; d < v->ndim; ++d) {
        if (v->shape[d] < 0) return DG_ERR_SHAPE;
        if (v->stride[d] < 0) return DG_ERR_STRIDE;
        if (v->shape[d] == 0) empty = true;
        int64_t *acc = d < v->row_dims ? &rows : &cols;
        if (!mul_ok(*acc, v->shape[d], acc)) return DG_ERR_SHAPE;
    }
    r.rows = rows;
    r.cols = cols;
    // byte span, with overflow checks
    int64_t span = 0;
    if (!empty) {
        for (int d = 0; d < v->ndim; ++d) {
            int64_t t;
            if (!mul_ok(v->shape[d] - 1, v->stride[d], &t) || !add_ok(span, t, &span)) return DG_ERR_STRIDE;
        }
        if (!add_ok(span, es, &span)) return DG_ERR_STRIDE;
    }
    r.span = span;
    if (!empty) {
        if (!v->ptr) return DG_ERR_NULL;
        if (reinterpret_cast<uintptr_t>(v->ptr) % es) return DG_ERR_ALIGN;
        for (int d = 0; d < v->ndim; ++d)
            if (v->shape[d] > 1 && v->stride[d] % es) return DG_ERR_ALIGN;
    }
    r.row = merge_group(v, 0, v->row_dims);
    r.col = merge_group(v, v->row_dims, v->ndim);

    if (is_output && !empty) {
        // no two elements may share an address: sorted by stride, every stride
        // must step over everything the smaller dims reach.
        int64_t sz[2 * kMaxDims], st[2 * kMaxDims];
        int n = 0;
        for (int i = 0; i < r.row.n; ++i) { sz[n] = r.row.size[i]; st[n] = r.row.stride[i]; ++n; }
        for (int i = 0; i < r.col.n; ++i) { sz[n] = r.col.size[i]; st[n] = r.col.stride[i]; ++n; }
        for (int i = 0; i < n; ++i)
            for (int j = i + 1; j < n; ++j)
                if (st[j] < st[i]) { std::swap(st[i], st[j]); std::swap(sz[i], sz[j]); }
        int64_t reach = es;  // bytes covered by the dims so far
        for (int i = 0; i < n; ++i) {
            if (st[i] < reach) return DG_ERR_STRIDE;
            int64_t t;
            if (!mul_ok(sz[i] - 1, st[i], &t) || !add_ok(t, reach, &reach)) return DG_ERR_STRIDE;
        }
    }

    // unit-stride group: a single merged dim of stride == element size
    if (r.col.n == 1 && r.col.stride[0] == es && r.row.n <= 1) r.unit_dim = 1;
    else if (r.row.n == 1 && r.row.stride[0] == es && r.col.n <= 1) r.unit_dim = 2;
    else if (r.col.n == 0 && r.row.n == 1 && r.row.stride[0] == es) r.unit_dim = 2;
    else if (r.row.n == 0 && r.col.n == 1 && r.col.stride[0] == es) r.unit_dim = 1;

    // Aligned vector width along a unit-stride innermost dim (for thread
    // loads): the run length, the base and every other stride must allow it.
    {
        const Axis *inner = nullptr, *other = nullptr;
        if (r.col.n >= 1 && r.col.stride[r.col.n - 1] == es) { inner = &r.col; other = &r.row; }
        else if (r.row.n >= 1 && r.row.stride[r.row.n - 1] == es) { inner = &r.row; other = &r.col; }
        int vb = es;
        if (inner) {
            vb = pow2_align(reinterpret_cast<uintptr_t>(v->ptr));
            vb = std::min(vb, pow2_align((uint64_t)(inner->size[inner->n - 1] * es)));
            for (int i = 0; i + 1 < inner->n; ++i) vb = std::min(vb, pow2_align((uint64_t)inner->stride[i]));
            for (int i = 0; i < other->n; ++i) vb = std::min(vb, pow2_align((uint64_t)other->stride[i]));
            vb = std::max(vb, es);
        }
        r.vec_bytes = vb;
    }

    // One 2-D TMA map: a unit-stride dim, the other group a single dim whose
    // stride is a multiple of 16 bytes, a 16-byte aligned base and extents
    // that fit the map's 32-bit dims.
    if (r.unit_dim != 0 && !empty) {
        const Axis &o = (r.unit_dim == 1) ? r.row : r.col;
        const int64_t inner_ext = (r.unit_dim == 1) ? cols : rows;
        const int64_t outer_ext = (r.unit_dim == 1) ? rows : cols;
        bool ok = (reinterpret_cast<uintptr_t>(v->ptr) % 16) == 0;
        if (o.n == 1) ok = ok && (o.stride[0] % 16 == 0) && o.stride[0] < (int64_t(1) << 40);
        ok = ok && inner_ext < (int64_t(1) << 31) && outer_ext < (int64_t(1) << 31);
        r.tma_ok = ok && o.n <= 1;
    }
    *info = r;
    return DG_OK;
}

}  // namespace dg

extern "C" dg_status dg_analyse_view(const dg_view *v, dg_view_info *out) {
    if (!v || !out) return DG_ERR_NULL;
    dg::ViewInfo r;
    dg_status st = dg::analyse(v, false, &r);
    if (st != DG_OK) return st;
    std::memset(out, 0, sizeof(*out));
    out->rows = r.rows;
    out->cols = r.cols;
    out->n_row = r.row.n;
    out->n_col = r.col.n;
    for (int i = 0; i < 4; ++i) {
        out->row_shape[i] = i < r.row.n ? r.row.size[i] : 1;
        out->row_stride[i] = i < r.row.n ? r.row.stride[i] : 0;
        out->col_shape[i] = i < r.col.n ? r.col.size[i] : 1;
        out->col_stride[i] = i < r.col.n ? r.col.stride[i] : 0;
    }
    out->unit_dim = r.unit_dim;
    out->tma_ok = r.tma_ok ? 1 : 0;
    out->span_bytes = r.span;
    out->vec_bytes = r.vec_bytes;
    return DG_OK;
}
