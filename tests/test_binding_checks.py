"""Host-side argument checks of the Python binding (CPU only): the C ABI sees
raw pointers, so a tensor that is too short for the shape the call implies
must be rejected in Python before any pointer reaches the library."""
import pytest
import torch

import speculative_decoding_block_spec_b200 as specv

E = torch.empty


def _block(B=3, L=4, V=64, K=None, packed_rows=None):
    d = dict(tokens=E(B, L, dtype=torch.int32), u=E(B, L), g=E(B, L + 1, V))
    d["draft"] = E(B, L, V) if K is None else E(B, K, L, V)
    d["target"] = E(B, L + 1, V) if packed_rows is None else E(packed_rows, V)
    return d


@pytest.mark.parametrize("case", [
    dict(),                                          # dense independent drafts
    dict(K=3),                                       # latent mixture
    dict(K=1),                                       # mixture layout with one category
    dict(L=0),                                       # empty block: g and target hold the bonus row only
    dict(packed_rows=20),                            # packed target rows with offsets
])
def test_valid_calls_pass(case):
    packed = case.get("packed_rows") is not None
    B, L, V = 3, case.get("L", 4), 64
    d = _block(B=B, L=L, V=V, K=case.get("K"), packed_rows=case.get("packed_rows"))
    K = case.get("K") or 1
    mix_w = E(B, K) if case.get("K") else None
    off = E(B + 1, dtype=torch.int32)[:B] if packed else None
    out = (E(B, dtype=torch.int32), E(B, L + 1, dtype=torch.int32))
    got = specv.check_verify_args(d["target"], d["draft"], d["tokens"], d["u"], d["g"], mix_w=mix_w,
                                  verify_len=E(B, dtype=torch.int32), target_row_off=off, out=out)
    assert got == (B, L, K, V)


@pytest.mark.parametrize("bad,msg", [
    (dict(target=E(3, 4, 64)), "target"),            # bonus row missing
    (dict(g=E(3, 4, 64)), "g"),                      # noise rows for positions 0..L-1 only
    (dict(g=E(3, 5, 63)), "g"),
    (dict(u=E(3, 3)), "u"),
    (dict(draft=E(3, 5, 64)), "draft"),
    (dict(tokens=E(3, 4, 1, dtype=torch.int32)), "tokens"),
])
def test_short_or_mismatched_tensors_are_rejected(bad, msg):
    d = _block()
    d.update(bad)
    with pytest.raises(ValueError, match=msg):
        specv.check_verify_args(d["target"], d["draft"], d["tokens"], d["u"], d["g"], mixture=False)
    # the wrappers check before touching the library or the device
    with pytest.raises(ValueError, match=msg):
        specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0)


def test_mixture_and_packed_and_outputs_are_checked():
    d = _block(K=2)
    with pytest.raises(ValueError, match="mix_w"):
        specv.spec_verify_mixture(d["target"], d["draft"], E(3, 3), d["tokens"], d["u"], d["g"], 1.0)
    p = _block(packed_rows=4)                        # fewer rows than one request's L+1 = 5
    with pytest.raises(ValueError, match="packed target"):
        specv.spec_verify_block(p["target"], p["draft"], p["tokens"], p["u"], p["g"], 1.0,
                                target_row_off=E(3, dtype=torch.int32))
    p = _block(packed_rows=20)
    with pytest.raises(ValueError, match="target_row_off"):
        specv.spec_verify_block(p["target"], p["draft"], p["tokens"], p["u"], p["g"], 1.0,
                                target_row_off=E(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="verify_len"):
        specv.spec_verify_block(d["target"], d["draft"][:, 0].contiguous(), d["tokens"], d["u"], d["g"], 1.0,
                                verify_len=E(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="out_tokens"):
        specv.spec_verify_block(d["target"], d["draft"][:, 0].contiguous(), d["tokens"], d["u"], d["g"], 1.0,
                                out=(E(3, dtype=torch.int32), E(3, 4, dtype=torch.int32)))


def test_tensors_on_different_devices_are_rejected():
    d = _block()
    with pytest.raises(ValueError, match="one device"):
        specv.check_verify_args(d["target"], d["draft"], d["tokens"], d["u"], E(3, 5, 64, device="meta"))


def test_dvl_and_softmax_shapes_are_checked():
    s = E(4, 6)
    with pytest.raises(ValueError, match="packed_target"):
        specv.dvl_allocate_pack(s, 10, dense_target=E(4, 7, 32), packed_target=E(9, 32))
    with pytest.raises(ValueError, match="dense_target"):
        specv.dvl_allocate_pack(s, 10, dense_target=E(4, 6, 32), packed_target=E(10, 32))
    with pytest.raises(ValueError, match="offsets"):
        specv.dvl_allocate_pack(s, 10, out=(E(4, dtype=torch.int32), E(4, dtype=torch.int32), None))
    x = E(5, 32)
    with pytest.raises(ValueError, match="row_lse"):
        specv.spec_softmax_T(x, 1.0, E(5), E(4))
    with pytest.raises(ValueError, match="probs"):
        specv.spec_softmax_T_noalloc(x, 1.0, E(5), E(5), probs=E(5, 31))
