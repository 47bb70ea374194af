"""Host logic of bench.py that needs no GPU: the kernel-source hash that keys
the recorded ncu traffic."""
import bench


def test_strip_comments_keeps_code_and_literals():
    src = 'int a = 1; // note\n/* block\n comment */ char b = \'/\';\n const char* s = "x//y /*z*/";\n\n  int c;'
    assert bench.strip_comments(src) == 'int a = 1; char b = \'/\'; const char* s = "x//y /*z*/"; int c;'


def test_hash_ignores_comments_and_layout_but_not_code():
    base = "__global__ void k(int* p) {\n  p[0] = 1;  // store\n}\n"
    assert bench.strip_comments(base) == bench.strip_comments(
        "// kernel\n__global__ void k(int* p) {\n\n  /* one */ p[0] = 1;\n}\n")
    assert bench.strip_comments(base) != bench.strip_comments("__global__ void k(int* p) {\n  p[0] = 2;\n}\n")


def test_recorded_traffic_matches_the_current_kernel_source():
    # the committed profiles were taken on this source; a kernel change makes
    # recorded_traffic return None until they are taken again
    assert bench.recorded_traffic("b2_h32_s4096_d128", "fp8/fp32") is not None
    assert bench.recorded_traffic("b2_h32_s4096_d128", "fp8/fp32+fp32") is not None
