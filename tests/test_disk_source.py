"""The disk stream source on the host, without a GPU: the device probe reads a file,
the acceptance rule refuses spinning and non-NVMe block devices and slow reads, the
`auto` choice takes memory when the store fits, and the file pool refuses misaligned
offsets, short staging and files shorter than their layers before it touches CUDA."""
import ctypes
import os

from nf4_layer_streamed_b200 import api, binding as B


def test_probe_reads_a_file(tmp_path):
    p = tmp_path / "store.bin"
    p.write_bytes(os.urandom(32 << 20))
    info = api.disk_probe(str(p), 16 << 20)
    assert info["read_gbs"] > 0
    assert set(info) == {"read_gbs", "block_device", "nvme", "rotational", "direct_io"}


def test_acceptance_rule():
    fast = 10.0
    assert api.disk_accept({"read_gbs": fast, "block_device": True, "nvme": True, "rotational": False}) == 0
    assert api.disk_accept({"read_gbs": fast, "block_device": False, "nvme": False, "rotational": False}) == 0
    # SATA SSD (a block device that is not NVMe), a spinning disk, a slow NVMe device
    assert api.disk_accept({"read_gbs": fast, "block_device": True, "nvme": False, "rotational": False}) == -10
    assert api.disk_accept({"read_gbs": fast, "block_device": True, "nvme": False, "rotational": True}) == -10
    assert api.disk_accept({"read_gbs": 0.4, "block_device": True, "nvme": True, "rotational": False}) == -10
    assert "refused" in B.last_error()


def test_auto_source_choice():
    assert api.choose_source(1 << 20) == "ram"
    assert api.choose_source(1 << 60) == "disk"


def test_file_pool_checks_arguments_on_host(tmp_path):
    p = tmp_path / "store.bin"
    p.write_bytes(bytes(3 * 4096))
    slots = ctypes.c_void_p(1 << 20)
    staging = ctypes.c_void_p(1 << 24)
    out = ctypes.c_void_p()
    sizes = (ctypes.c_size_t * 3)(4000, 4000, 4000)

    def create(offs, path=str(p), st_bytes=8192, depth=2):
        o = (ctypes.c_size_t * 3)(*offs)
        return B.call_status("nf4ls_pool_create_file", path.encode(), ctypes.cast(o, ctypes.c_void_p),
                             ctypes.cast(sizes, ctypes.c_void_p), 3, depth, slots, 4096, staging, st_bytes,
                             ctypes.byref(out))

    assert B.lib().nf4ls_pool_file_staging_bytes(ctypes.cast(sizes, ctypes.c_void_p), 3) == 8192
    assert create((0, 256, 8192)) == -3                    # offsets must be 4096-aligned
    assert create((0, 4096, 8192), st_bytes=4096) == -3    # staging below 2 x 4096
    assert create((0, 4096, 8192), depth=1) == -1
    assert create((0, 4096, 8192), path=str(tmp_path / "missing.bin")) == -11
    assert create((0, 4096, 12288)) == -1                  # the last layer ends past the file
