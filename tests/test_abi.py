"""The C ABI library loads, exports every symbol include/bitlinear.h
declares, and rejects bad arguments on the host (no device work: every check
here returns before the library touches CUDA)."""
import ctypes
import os
import re

import pytest

import ternary_weight_w1_b200 as bl

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "bitlinear.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(bl.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = bl.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    assert bl.status_string(bl.BITLINEAR_OK) == "ok"
    assert bl.status_string(bl.BITLINEAR_ERR_TIMEOUT) == "device wait timed out"
    assert bl.status_string(bl.BITLINEAR_ERR_HOST) == "host allocation failed"
    assert bl.status_string(99) == "unknown status"


def test_binding_status_codes_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    enum = re.search(r"typedef enum \{(.*?)\} bitlinear_status;", text, flags=re.S).group(1)
    codes = dict((k, int(v)) for k, v in re.findall(r"(BITLINEAR_\w+)\s*=\s*(\d+)", enum))
    assert len(codes) >= 10
    for name, value in codes.items():
        assert getattr(bl, name) == value, name
        assert bl.status_string(value) != "unknown status", name


def test_packed_bytes():
    assert bl.bitlinear_packed_bytes(6912, 2560) == 6912 * 640
    assert bl.bitlinear_packed_bytes(1, 128) == 16 * 32          # one padded row block
    assert bl.bitlinear_packed_bytes(17, 256) == 32 * 64
    assert bl.bitlinear_packed_bytes(0, 256) == 0
    assert bl.bitlinear_packed_bytes(4, 64) == 0
    assert bl.bitlinear_packed_bytes(4, 200) == 0


def test_workspace_bytes():
    assert bl.bitlinear_workspace_bytes(1, 6912, 2560) == 0          # GEMV
    assert bl.bitlinear_workspace_bytes(2048, 6912, 2560) >= 2048 * 2560 + 2 * 2048 * 4
    assert bl.bitlinear_workspace_bytes(1, 6912, 2560, bl.PATH_TC) >= 2560 + 8
    assert bl.bitlinear_workspace_bytes(4, 64, 100) == ctypes.c_size_t(-1).value
    assert bl.bitlinear_workspace_bytes(0, 64, 256) == 0
    # the automatic GEMV path also needs x~ of all tokens in shared memory
    # (M * K <= 196608): six tokens of K = 32768 fit, of K = 65536 do not
    assert bl.bitlinear_workspace_bytes(6, 128, 32768) == 0
    assert bl.bitlinear_workspace_bytes(6, 128, 65536) >= 6 * 65536
    assert bl.bitlinear_workspace_bytes(7, 128, 256) > 0


FAKE = 1 << 20          # a 16-byte-aligned non-null address; never dereferenced


def fwd(**kw):
    a = dict(x=FAKE, xdt=0, M=1, K=256, packed=FAKE, gamma=1.0, N=64, y=FAKE, ws=None,
             wsb=0, stream=None, acc=None, xq=None, beta=None)
    a.update(kw)
    return bl.lib().bitlinear_forward(a["x"], a["xdt"], a["M"], a["K"], a["packed"], a["gamma"],
                                      a["N"], a["y"], a["ws"], a["wsb"], a["stream"], a["acc"],
                                      a["xq"], a["beta"])


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), bl.BITLINEAR_ERR_ARG),
    (dict(packed=None), bl.BITLINEAR_ERR_ARG),
    (dict(y=None), bl.BITLINEAR_ERR_ARG),
    (dict(M=-1), bl.BITLINEAR_ERR_ARG),
    (dict(N=0), bl.BITLINEAR_ERR_ARG),
    (dict(K=200), bl.BITLINEAR_ERR_SHAPE),
    (dict(K=64), bl.BITLINEAR_ERR_SHAPE),
    (dict(K=65536 + 128), bl.BITLINEAR_ERR_SHAPE),
    (dict(xdt=7), bl.BITLINEAR_ERR_DTYPE),
    (dict(x=FAKE + 8), bl.BITLINEAR_ERR_ALIGN),
    (dict(packed=FAKE + 4), bl.BITLINEAR_ERR_ALIGN),
    (dict(y=FAKE + 2), bl.BITLINEAR_ERR_ALIGN),
    (dict(xq=FAKE + 1), bl.BITLINEAR_ERR_ALIGN),
    (dict(acc=FAKE + 2), bl.BITLINEAR_ERR_ALIGN),
    (dict(M=0), bl.BITLINEAR_OK),                 # empty batch: nothing to do
    (dict(M=0, x=None, y=None), bl.BITLINEAR_OK),
])
def test_forward_rejects_bad_arguments(kw, status):
    assert fwd(**kw) == status


def test_forward_ex_rejects_bad_path():
    L = bl.lib()
    rc = L.bitlinear_forward_ex(FAKE, 0, 1, 256, FAKE, 1.0, 64, FAKE, None, 0, None, None,
                                None, None, 9)
    assert rc == bl.BITLINEAR_ERR_ARG


def fwd_norm(**kw):
    a = dict(x=FAKE, xdt=0, M=1, K=256, g=FAKE, eps=2.0 ** -23, packed=FAKE, gamma=1.0, N=64,
             y=FAKE, ws=None, wsb=0, stream=None, acc=None, xq=None, beta=None, path=0)
    a.update(kw)
    return bl.lib().bitlinear_forward_rmsnorm(a["x"], a["xdt"], a["M"], a["K"], a["g"], a["eps"],
                                              a["packed"], a["gamma"], a["N"], a["y"], a["ws"],
                                              a["wsb"], a["stream"], a["acc"], a["xq"], a["beta"],
                                              a["path"])


@pytest.mark.parametrize("kw,status", [
    (dict(g=None), bl.BITLINEAR_ERR_ARG),             # gains required for a non-empty batch
    (dict(g=FAKE + 4), bl.BITLINEAR_ERR_ALIGN),
    (dict(eps=0.0), bl.BITLINEAR_ERR_ARG),
    (dict(eps=-1e-6), bl.BITLINEAR_ERR_ARG),
    (dict(eps=float("nan")), bl.BITLINEAR_ERR_ARG),
    (dict(eps=float("inf")), bl.BITLINEAR_ERR_ARG),
    (dict(K=200), bl.BITLINEAR_ERR_SHAPE),            # the forward's own checks follow
    (dict(x=None), bl.BITLINEAR_ERR_ARG),
    (dict(y=FAKE + 2), bl.BITLINEAR_ERR_ALIGN),
    (dict(path=9), bl.BITLINEAR_ERR_ARG),
    (dict(M=0, g=None), bl.BITLINEAR_OK),             # empty batch: nothing to do
])
def test_forward_rmsnorm_rejects_bad_arguments(kw, status):
    assert fwd_norm(**kw) == status


def test_gemv_admits_what_its_shared_memory_holds():
    # x~ (M * K bytes) must fit beside the GEMV's other shared memory: at
    # most 196608 bytes for every token tile. Only host-side calls here: the
    # sizing function, and forward calls whose shape is refused before any
    # device work.
    size_max = ctypes.c_size_t(-1).value

    def gemv_ok(M, K):
        return bl.bitlinear_workspace_bytes(M, 64, K, bl.PATH_GEMV) != size_max
    assert gemv_ok(16, 12288)                     # 196608
    assert not gemv_ok(16, 12416)                 # 198656
    assert gemv_ok(12, 16384)
    assert not gemv_ok(12, 16512)
    assert gemv_ok(8, 24576)
    assert gemv_ok(3, 65536)
    assert not gemv_ok(17, 128)
    L = bl.lib()
    rc = L.bitlinear_forward_ex(FAKE, 0, 16, 12416, FAKE, 1.0, 64, FAKE, None, 0, None, None,
                                None, None, bl.PATH_GEMV)
    assert rc == bl.BITLINEAR_ERR_SHAPE
    # a group is one launch: its largest x~ must fit
    big4, small16 = (FAKE, 4, 49280, 64, FAKE, FAKE), (FAKE, 16, 128, 64, FAKE, FAKE)
    assert grouped([big4, small16]) == bl.BITLINEAR_ERR_SHAPE

def test_quant_act_rejects_bad_arguments():
    L = bl.lib()
    assert L.bitlinear_quant_act(None, 0, 2, 256, FAKE, FAKE, None) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_quant_act(FAKE, 0, 2, 200, FAKE, FAKE, None) == bl.BITLINEAR_ERR_SHAPE
    assert L.bitlinear_quant_act(FAKE, 3, 2, 256, FAKE, FAKE, None) == bl.BITLINEAR_ERR_DTYPE
    assert L.bitlinear_quant_act(FAKE, 0, 2, 256, FAKE + 1, FAKE, None) == bl.BITLINEAR_ERR_ALIGN
    assert L.bitlinear_quant_act(FAKE, 0, 0, 256, FAKE, FAKE, None) == bl.BITLINEAR_OK


def test_inject_timeout_rejects_bad_limit():
    L = bl.lib()
    rc = L.bitlinear_forward_inject_timeout(FAKE, 0, 1, 256, FAKE, 1.0, 64, FAKE, FAKE, 4096,
                                            None, bl.PATH_TC, 0)
    assert rc == bl.BITLINEAR_ERR_ARG
    # only an explicit kernel choice is accepted
    for path in (bl.PATH_AUTO, 3, -1):
        rc = L.bitlinear_forward_inject_timeout(FAKE, 0, 1, 256, FAKE, 1.0, 64, FAKE, FAKE, 4096,
                                                None, path, 1000)
        assert rc == bl.BITLINEAR_ERR_ARG


def test_get_fault_rejects_null():
    assert bl.lib().bitlinear_get_fault(None, None) == bl.BITLINEAR_ERR_ARG


def grouped(problems, xdt=0):
    arr = (bl._Problem * max(1, len(problems)))()
    for i, (x, M, K, N, packed, y) in enumerate(problems):
        arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
    return bl.lib().bitlinear_forward_grouped(ctypes.addressof(arr), len(problems), xdt, None)


def test_grouped_rejects_bad_arguments():
    good = (FAKE, 1, 256, 64, FAKE, FAKE)
    assert bl.lib().bitlinear_forward_grouped(None, 1, 0, None) == bl.BITLINEAR_ERR_ARG
    assert grouped([]) == bl.BITLINEAR_ERR_ARG
    assert grouped([good] * 9) == bl.BITLINEAR_ERR_ARG
    assert grouped([good, (FAKE, 1, 200, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert grouped([good, (FAKE, 17, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert grouped([good, (FAKE, 16, 16384, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert grouped([good, (None, 1, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ARG
    assert grouped([good, (FAKE + 8, 1, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ALIGN
    assert grouped([good], xdt=5) == bl.BITLINEAR_ERR_DTYPE
    assert grouped([(None, 0, 256, 64, None, None)]) == bl.BITLINEAR_OK   # only empty problems


def grouped_host(problems, xdt=0, x_host=FAKE, y_host=FAKE):
    arr = (bl._Problem * max(1, len(problems)))()
    for i, (x, M, K, N, packed, y) in enumerate(problems):
        arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
    return bl.lib().bitlinear_forward_grouped_host(ctypes.addressof(arr), len(problems), xdt,
                                                   x_host, y_host, None)


def test_grouped_b3_rejects_bad_arguments():
    def call(problems, xdt=0):
        arr = (bl._Problem * max(1, len(problems)))()
        for i, (x, M, K, N, packed, y) in enumerate(problems):
            arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
        return bl.lib().bitlinear_forward_grouped_b3(ctypes.addressof(arr), len(problems), xdt,
                                                     None)
    good = (FAKE, 1, 256, 64, FAKE, FAKE)
    assert bl.lib().bitlinear_forward_grouped_b3(None, 1, 0, None) == bl.BITLINEAR_ERR_ARG
    assert call([]) == bl.BITLINEAR_ERR_ARG
    assert call([good] * 9) == bl.BITLINEAR_ERR_ARG
    assert call([good, (FAKE, 17, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    # 16 x 12288 is within the 2-bit GEMV's limit (196608), but the base-3
    # rows pad to 12320
    assert call([(FAKE, 16, 12288, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert call([good, (FAKE + 8, 1, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ALIGN
    assert call([good], xdt=5) == bl.BITLINEAR_ERR_DTYPE
    assert call([(None, 0, 256, 64, None, None)]) == bl.BITLINEAR_OK   # nothing to do


def test_grouped_host_rejects_bad_arguments():
    """The host-buffer call checks what bitlinear_forward_grouped checks, and
    its host buffers, before any copy or launch."""
    good = (FAKE, 1, 256, 64, FAKE, FAKE)
    assert bl.lib().bitlinear_forward_grouped_host(None, 1, 0, FAKE, FAKE, None) == \
        bl.BITLINEAR_ERR_ARG
    assert grouped_host([]) == bl.BITLINEAR_ERR_ARG
    assert grouped_host([good] * 9) == bl.BITLINEAR_ERR_ARG
    assert grouped_host([good, (FAKE, 17, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert grouped_host([good, (FAKE + 8, 1, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ALIGN
    assert grouped_host([good], xdt=5) == bl.BITLINEAR_ERR_DTYPE
    assert grouped_host([good], x_host=None) == bl.BITLINEAR_ERR_ARG
    assert grouped_host([good], y_host=None) == bl.BITLINEAR_ERR_ARG
    assert grouped_host([(None, 0, 256, 64, None, None)]) == bl.BITLINEAR_OK   # nothing to do


def test_grouped_host_call_refuses_device_or_wrong_host_buffers():
    """The prepared binding checks the host tensors' place, dtype and size
    before its library call (no GPU needed: the problem list is built from
    shapes alone and never reaches the library here)."""
    import torch
    x = torch.zeros(256, dtype=torch.bfloat16)
    y = torch.zeros(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="elements"):
        bl._host_buffer(torch.zeros(255, dtype=torch.bfloat16), "x_host", torch.bfloat16, 256)
    with pytest.raises(TypeError, match="must be"):
        bl._host_buffer(torch.zeros(256, dtype=torch.float32), "x_host", torch.bfloat16, 256)
    with pytest.raises(ValueError, match="contiguous"):
        bl._host_buffer(torch.zeros(512, dtype=torch.bfloat16)[::2], "x_host", torch.bfloat16,
                        256)
    assert bl._host_buffer(x, "x_host", torch.bfloat16, 256) == x.data_ptr()
    assert bl._host_buffer(y, "y_host", torch.bfloat16, 64) == y.data_ptr()
    with pytest.raises(ValueError, match="y_dev"):
        bl.GroupedHostCall([(x.view(1, -1), None, 1.0, 64, None)])


def grouped_ws(problems, xdt=0, ws=FAKE, ws_bytes=1 << 30):
    arr = (bl._Problem * max(1, len(problems)))()
    for i, (x, M, K, N, packed, y) in enumerate(problems):
        arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
    return bl.lib().bitlinear_forward_grouped_ws(ctypes.addressof(arr), len(problems), xdt, ws,
                                                 ws_bytes, None)


def grouped_ws_bytes(problems):
    arr = (bl._Problem * max(1, len(problems)))()
    for i, (x, M, K, N, packed, y) in enumerate(problems):
        arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
    return bl.lib().bitlinear_workspace_bytes_grouped(ctypes.addressof(arr), len(problems))


def test_grouped_ws_rejects_bad_arguments():
    good = (FAKE, 8, 256, 64, FAKE, FAKE)
    assert bl.lib().bitlinear_forward_grouped_ws(None, 1, 0, FAKE, 1, None) == bl.BITLINEAR_ERR_ARG
    assert grouped_ws([]) == bl.BITLINEAR_ERR_ARG
    assert grouped_ws([good] * 9) == bl.BITLINEAR_ERR_ARG
    assert grouped_ws([good, (FAKE, 8, 200, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_SHAPE
    assert grouped_ws([good, (None, 8, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ARG
    assert grouped_ws([good, (FAKE + 8, 8, 256, 64, FAKE, FAKE)]) == bl.BITLINEAR_ERR_ALIGN
    assert grouped_ws([good], xdt=5) == bl.BITLINEAR_ERR_DTYPE
    assert grouped_ws([(None, 0, 256, 64, None, None)]) == bl.BITLINEAR_OK   # only empty problems


def test_grouped_ws_bytes():
    size_max = ctypes.c_size_t(-1).value
    small = [(None, 1, 2560, 6912, None, None), (None, 6, 6912, 2560, None, None)]
    assert grouped_ws_bytes(small) == 0                       # one GEMV launch
    big = [(None, 8, 2560, 6912, None, None), (None, 8, 6912, 2560, None, None)]
    need = grouped_ws_bytes(big)
    assert need >= 8 * 2560 + 8 * 6912 + 4 * 8 * 4
    assert need >= grouped_ws_bytes(big[:1])
    assert grouped_ws_bytes([(None, 8, 200, 64, None, None)]) == size_max
    assert grouped_ws_bytes([]) == size_max


def test_binding_refuses_host_tensors():
    # a host tensor handed to a kernel would make it read host addresses:
    # the binding refuses it before any library call (no GPU needed)
    import torch
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    packed = torch.zeros((bl.bitlinear_packed_bytes(64, 256),), dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bl.bitlinear_quant_act(x, xq=x.to(torch.int8), beta=torch.zeros(4))
    with pytest.raises(ValueError, match="CUDA tensor"):
        bl.bitlinear_forward(x, packed, 1.0, 64, y=torch.zeros((4, 64), dtype=torch.bfloat16),
                             path=bl.PATH_GEMV)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bl.bitlinear_forward_grouped([(x, packed, 1.0, 64,
                                       torch.zeros((4, 64), dtype=torch.bfloat16))])
    with pytest.raises(ValueError, match="CUDA tensor"):
        bl.bitlinear_forward_rmsnorm(x, packed, 1.0, 64, torch.ones(256),
                                     y=torch.zeros((4, 64), dtype=torch.bfloat16),
                                     path=bl.PATH_GEMV)


def ffn(M=1, K=256, F=512, x=FAKE, gp=FAKE, up=FAKE, dp=FAKE, gg=None, ug=None, dg=None,
        eps=2.0 ** -23, h=FAKE, y=FAKE, ws=None, ws_bytes=0, xdt=0):
    return bl.lib().bitlinear_ffn_forward(x, xdt, M, K, F, gp, 1.0, up, 1.0, dp, 1.0, gg, ug, dg,
                                          eps, h, y, ws, ws_bytes, None, None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(gg=FAKE), bl.BITLINEAR_ERR_ARG),             # gate gains without up gains
    (dict(ug=FAKE), bl.BITLINEAR_ERR_ARG),
    (dict(K=200), bl.BITLINEAR_ERR_SHAPE),
    (dict(F=1000), bl.BITLINEAR_ERR_SHAPE),
    (dict(M=17), bl.BITLINEAR_ERR_WORKSPACE),           # gate/up on the tensor cores
    (dict(M=4, K=65536, F=128), bl.BITLINEAR_ERR_WORKSPACE),   # x~ beyond the GEMV's limit
    (dict(M=6, K=32768, gg=FAKE, ug=FAKE), bl.BITLINEAR_ERR_WORKSPACE),  # two copies of x~
    (dict(M=1, K=65664), bl.BITLINEAR_ERR_SHAPE),       # K beyond 65536
    (dict(M=-1), bl.BITLINEAR_ERR_ARG),
    (dict(xdt=7), bl.BITLINEAR_ERR_DTYPE),
    (dict(dg=FAKE, eps=0.0), bl.BITLINEAR_ERR_ARG),
    (dict(gg=FAKE, ug=FAKE, eps=float("nan")), bl.BITLINEAR_ERR_ARG),
    (dict(h=None), bl.BITLINEAR_ERR_ARG),
    (dict(dp=None), bl.BITLINEAR_ERR_ARG),
    (dict(h=FAKE + 4), bl.BITLINEAR_ERR_ALIGN),
    (dict(y=FAKE + 2), bl.BITLINEAR_ERR_ALIGN),
    (dict(dg=FAKE + 4), bl.BITLINEAR_ERR_ALIGN),
    (dict(M=12, K=2560, F=6912), bl.BITLINEAR_ERR_WORKSPACE),   # down projection on tensor cores
    (dict(M=0, x=None, h=None, y=None), bl.BITLINEAR_OK),       # empty batch: nothing to do
])
def test_ffn_forward_rejects_bad_arguments(kw, status):
    assert ffn(**kw) == status


def test_ffn_workspace():
    """Decode batches: the down projection's workspace (0 on the GEMV).
    Larger batches: at least the gate/up group's scratch plus its two bf16
    outputs, and at least the down projection's."""
    size_max = ctypes.c_size_t(-1).value
    assert bl.bitlinear_workspace_bytes_ffn(1, 2560, 6912) == 0
    assert (bl.bitlinear_workspace_bytes_ffn(6, 2560, 6912) ==
            bl.bitlinear_workspace_bytes(6, 2560, 6912))
    for M in (7, 12, 17, 300):
        need = bl.bitlinear_workspace_bytes_ffn(M, 2560, 6912)
        assert need >= bl.bitlinear_workspace_bytes(M, 2560, 6912)
        assert need >= 2 * M * 6912 * 2 + M * 2560
    assert bl.bitlinear_workspace_bytes_ffn(1, 2560, 1000) == size_max
    assert bl.bitlinear_workspace_bytes_ffn(-1, 2560, 6912) == size_max


def test_grouped_rmsnorm_rejects_bad_arguments():
    L = bl.lib()
    good = (FAKE, 1, 256, 64, FAKE, FAKE)

    def call(problems, gains, eps=2.0 ** -23, count=None):
        arr = (bl._Problem * max(1, len(problems)))()
        for i, (x, M, K, N, packed, y) in enumerate(problems):
            arr[i] = bl._Problem(x, M, K, N, packed, 1.0, y)
        g = None if gains is None else (ctypes.c_void_p * max(1, len(gains)))(*gains)
        n = len(problems) if count is None else count
        return L.bitlinear_forward_grouped_rmsnorm(ctypes.addressof(arr),
                                                   None if g is None else ctypes.addressof(g),
                                                   n, eps, 0, None, 0, None)
    assert call([good], None) == bl.BITLINEAR_ERR_ARG              # no gains array
    assert call([good], [None]) == bl.BITLINEAR_ERR_ARG            # a missing gain
    assert call([good], [FAKE + 4]) == bl.BITLINEAR_ERR_ALIGN
    assert call([good], [FAKE], eps=0.0) == bl.BITLINEAR_ERR_ARG
    assert call([good], [FAKE], eps=float("inf")) == bl.BITLINEAR_ERR_ARG
    assert call([good], [FAKE], count=0) == bl.BITLINEAR_ERR_ARG
    assert call([good] * 9, [FAKE] * 9) == bl.BITLINEAR_ERR_ARG
    assert call([(FAKE, 1, 200, 64, FAKE, FAKE)], [FAKE]) == bl.BITLINEAR_ERR_SHAPE
    # an empty batch needs no gain and does nothing
    assert call([(FAKE, 0, 256, 64, FAKE, FAKE)], [None]) == bl.BITLINEAR_OK


def test_forward_b3_rejects_bad_arguments():
    L = bl.lib()

    def call(M=1, K=256, N=64, x=FAKE, packed=FAKE, y=FAKE, xdt=0):
        return L.bitlinear_forward_b3(x, xdt, M, K, packed, 1.0, N, y, None, None, None, None)
    assert call(x=None) == bl.BITLINEAR_ERR_ARG
    assert call(K=200) == bl.BITLINEAR_ERR_SHAPE
    assert call(M=17) == bl.BITLINEAR_ERR_SHAPE                 # the GEMV path only
    assert call(M=16, K=12288) == bl.BITLINEAR_ERR_SHAPE        # padded x~ 16 * 12320 bytes
    assert call(xdt=3) == bl.BITLINEAR_ERR_DTYPE
    assert call(y=FAKE + 2) == bl.BITLINEAR_ERR_ALIGN
    assert call(M=0, x=None, y=None) == bl.BITLINEAR_OK
