// qrx_check.cuh -- bounds-checked builds.
//
// Built with -DQRX_CHECK (libqrx_check.so), the kernels test every index that
// comes from data rather than from their own loop bounds (permutation
// positions, token rows taken from `sorted`, output rows derived from
// `offsets`, `inv` entries) against the sizes they were given.  A miss records
// DERR_BOUNDS in the sticky device status, which qrx_last_error reports as
// QRX_EDEVICE, and the access is skipped or clamped, so a checked run never
// touches memory outside its buffers.  In the default build both macros
// expand to nothing and the kernels' code is unchanged.
//
//   QRX_CHECK_OR(ok, action);    if !ok: raise DERR_BOUNDS, then run `action`
//                                (continue, return, or a clamp)
//   QRX_CHECK_ONLY(decl...);     code that exists only in checked builds
//                                (the bounds the checks compare against)
#pragma once

#ifdef QRX_CHECK
#define QRX_CHECK_OR(ok, action)                 \
    if (!(ok)) {                                 \
        ::qrx::raise_status(::qrx::DERR_BOUNDS); \
        action;                                  \
    } else                                       \
        (void)0
#define QRX_CHECK_ONLY(...) __VA_ARGS__
#else
#define QRX_CHECK_OR(ok, action) (void)0
#define QRX_CHECK_ONLY(...)
#endif
