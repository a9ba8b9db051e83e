"""The workspace-free importance entry point (hinm_importance_noalloc) against the
workspace one (hinm_importance): bit-identical I on two calls in a row.

The second call uses other inputs and a different K, so a scratch value left over from
the first call, or one read before it is written, would show as a mismatch.  The file
is named to be collected last; it builds its own inputs and passes alone too.
"""
import ctypes

import numpy as np
import pytest

import hinm_inputs as hi

torch = pytest.importorskip("torch")

MAX_K = 16384  # channels the static scratch holds


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def both_paths(H, w):
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    I_ws = H.hinm_importance(W, X)
    I_na = torch.full((w.M, w.K), float("nan"), dtype=torch.float32, device="cuda")
    H.hinm_importance_noalloc(W, X, I_na)
    torch.cuda.synchronize()
    return I_ws.cpu().numpy().view(np.uint32), I_na.cpu().numpy().view(np.uint32)


@pytest.mark.gpu
@pytest.mark.parametrize("shapes", [
    ((256, 1024, 64), (128, 200, 40)),        # second call: smaller, ragged K and N
    ((128, 196, 24), (192, MAX_K, 16)),       # second call: the largest K the scratch holds
])
def test_noalloc_matches_workspace_entry_two_calls(H, shapes):
    for call, (M, K, N) in enumerate(shapes):
        w = hi.custom(M, K, N, 64, seed=9100 + 7 * call + K, t_s=0.5, v_s=0.2)
        ref, got = both_paths(H, w)
        np.testing.assert_array_equal(got, ref, err_msg=f"call {call}: M={M} K={K} N={N}")


@pytest.mark.gpu
def test_noalloc_same_stream_back_to_back(H):
    """Two calls queued on one stream with no host sync between them."""
    a = hi.custom(128, 4096, 32, 64, seed=9201, t_s=0.5, v_s=0.2)
    b = hi.custom(128, 2048, 48, 64, seed=9202, t_s=0.5, v_s=0.2)
    Wa, Xa, Wb, Xb = (dev_bf16(x) for x in (a.W_bits, a.X_bits, b.W_bits, b.X_bits))
    Ia_ref, Ib_ref = H.hinm_importance(Wa, Xa), H.hinm_importance(Wb, Xb)
    Ia = torch.empty((a.M, a.K), dtype=torch.float32, device="cuda")
    Ib = torch.empty((b.M, b.K), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        H.hinm_importance_noalloc(Wa, Xa, Ia, stream=s)
        H.hinm_importance_noalloc(Wb, Xb, Ib, stream=s)
    s.synchronize()
    np.testing.assert_array_equal(Ia.cpu().numpy().view(np.uint32),
                                  Ia_ref.cpu().numpy().view(np.uint32))
    np.testing.assert_array_equal(Ib.cpu().numpy().view(np.uint32),
                                  Ib_ref.cpu().numpy().view(np.uint32))


def test_noalloc_rejects_k_beyond_scratch():
    """K above the static scratch is refused on the host, before any device access."""
    from conftest import build_library
    build_library()
    import pruning_hinm_spmm_b200 as H
    lib = ctypes.CDLL(H.LIB_PATH)
    lib.hinm_importance_noalloc.restype = ctypes.c_int
    lib.hinm_importance_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p]
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    HINM_ERR_SHAPE = 2
    assert lib.hinm_importance_noalloc(fake, fake, 64, MAX_K + 4, 16, fake, None) == HINM_ERR_SHAPE
    assert lib.hinm_importance_noalloc(fake, fake, 64, MAX_K + 4096, 16, fake, None) == HINM_ERR_SHAPE
